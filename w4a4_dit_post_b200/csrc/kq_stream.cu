// Streaming kernels of the online quantizer: kq_quantize, kq_transform and
// the SmoothQuant comparison quantizer sq_quantize.
//
// Data view.  Rows are contiguous and d is a multiple of 32, so an [M][d]
// activation is a flat array of M*d/32 blocks of 32 elements; block g is
// token g / nb, channel block j = g % nb.  Its 16 code bytes sit at
// codes + 16 g and its scale byte at scales + g, so one thread per block
// writes coalesced 16-byte and 1-byte stores.
//
// Pipeline.  A persistent grid (a whole number of CTAs per SM); each CTA
// walks tiles of 256 blocks (one per thread).  Thread 0 keeps kStages tiles
// in flight with 2-D TMA loads (box = 32 elements x 256 blocks) into
// swizzled shared memory, each stage guarded by an mbarrier.  The swizzle
// (64-byte for bf16 rows, 128-byte for fp32 rows) makes the per-thread
// 16-byte reads of a whole 64/128-byte block conflict-free.  After reading
// its block into registers a thread joins a CTA barrier, and thread 0 reuses
// the stage for the tile kStages ahead; the transform, the encoding and the
// stores then overlap the loads in flight.
//
// Per-block coefficients are built once per CTA in shared memory: for
// KroQuant 5 factors x (A00, A01, A10, A11) from the 15 LU parameters; for
// SmoothQuant the 32 inverse scales.  Row strides of 80 and 144 bytes (5 and
// 9 16-byte units, odd) keep 8 consecutive blocks on distinct bank groups.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "kq.h"
#include "kq_device.cuh"
#include "kq_host.h"

namespace kq {

// Per-device status word (KQ_DEVSTAT_* bits); each device that loads this
// module holds its own copy.
__device__ unsigned int g_devstat = 0;

constexpr int kThreads = 256;
constexpr int kTileBlocks = 256;   // blocks per tile = TMA box rows

enum class Op : int { kKqQuant = 0, kKqTransform = 1, kSqQuant = 2 };

template <int kInBytes>
struct InLayout;

template <>
struct InLayout<2> {                     // bf16: 64-byte block rows, 64B swizzle
  static constexpr int kBlockBytes = 64;
  static constexpr int kChunks = 4;      // 16-byte chunks per block
  __device__ static int swz(int t) { return (t >> 1) & 3; }
};

template <>
struct InLayout<4> {                     // fp32: 128-byte block rows, 128B swizzle
  static constexpr int kBlockBytes = 128;
  static constexpr int kChunks = 8;
  __device__ static int swz(int t) { return t & 7; }
};

template <Op kOp>
struct TableLayout {
  // floats per coefficient row (padded to an odd number of 16-byte units)
  static constexpr int kRowFloats = (kOp == Op::kSqQuant) ? 36 : 20;
};

template <int kInBytes, Op kOp>
struct StreamCfg {
  static constexpr int kStages = (kInBytes == 2) ? 4 : 2;
  static constexpr int kStageBytes = kTileBlocks * InLayout<kInBytes>::kBlockBytes;
  static constexpr int kBarOffset = kStages * kStageBytes;
  static constexpr int kTableOffset = kBarOffset + 128;
  static size_t smem_bytes(int nb) {
    // + 1024 for aligning the dynamic base to the 1024-byte swizzle atom
    return 1024 + kTableOffset + (size_t)nb * TableLayout<kOp>::kRowFloats * sizeof(float);
  }
};

template <int kInBytes>
__device__ __forceinline__ void load_block(const uint8_t* stage, int tid, float2 (&v)[16]) {
  using L = InLayout<kInBytes>;
  const uint8_t* row = stage + tid * L::kBlockBytes;
  const int sw = L::swz(tid);
  uint4 q[L::kChunks];
#pragma unroll
  for (int c = 0; c < L::kChunks; ++c)
    q[c] = *reinterpret_cast<const uint4*>(row + ((c ^ sw) << 4));
  if constexpr (kInBytes == 2) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      v[4 * c + 0] = bf16x2_to_float2(q[c].x);
      v[4 * c + 1] = bf16x2_to_float2(q[c].y);
      v[4 * c + 2] = bf16x2_to_float2(q[c].z);
      v[4 * c + 3] = bf16x2_to_float2(q[c].w);
    }
  } else {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      v[2 * c + 0] = make_float2(__uint_as_float(q[c].x), __uint_as_float(q[c].y));
      v[2 * c + 1] = make_float2(__uint_as_float(q[c].z), __uint_as_float(q[c].w));
    }
  }
}

template <int kInBytes, Op kOp>
__global__ void __launch_bounds__(kThreads, 2)
stream_kernel(const __grid_constant__ CUtensorMap tmap, const float* __restrict__ coef_src,
              int nb, int n_blocks, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
              float* __restrict__ y_out) {
  using Cfg = StreamCfg<kInBytes, kOp>;
  constexpr int kStages = Cfg::kStages;
  constexpr int kRow = TableLayout<kOp>::kRowFloats;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOffset);
  int* abort_flag = reinterpret_cast<int*>(smem + Cfg::kBarOffset + 8 * kStages);
  float* table = reinterpret_cast<float*>(smem + Cfg::kTableOffset);

  const int tid = threadIdx.x;
  const int n_tiles = (n_blocks + kTileBlocks - 1) / kTileBlocks;

  if (tid == 0) {
    tma_prefetch_desc(&tmap);
#pragma unroll
    for (int s = 0; s < kStages; ++s) mbar_init(smem_addr(&bars[s]), 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  __syncthreads();
  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
      const int tile = blockIdx.x + s * gridDim.x;
      if (tile < n_tiles) {
        mbar_arrive_expect_tx(smem_addr(&bars[s]), Cfg::kStageBytes);
        tma_load_2d(smem_addr(smem + s * Cfg::kStageBytes), &tmap, 0, tile * kTileBlocks,
                    smem_addr(&bars[s]));
      }
    }
  }

  // coefficient table (overlaps the first loads)
  if constexpr (kOp == Op::kSqQuant) {
    for (int i = tid; i < nb * 32; i += kThreads)
      table[(i >> 5) * kRow + (i & 31)] = coef_src[i];
  } else {
    for (int i = tid; i < nb * 5; i += kThreads) {
      const int j = i / 5, m = i - 5 * j;
      const float* p = coef_src + 15 * j + 3 * m;
      *reinterpret_cast<float4*>(table + j * kRow + 4 * m) = lu_factor(p[0], p[1], p[2]);
    }
  }
  __syncthreads();

  const int step = kTileBlocks * gridDim.x;       // blocks between a thread's tiles
  const int jstep = step % nb;
  int j = (blockIdx.x * kTileBlocks + tid) % nb;  // channel block of this thread's block

  int k = 0;
  for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++k) {
    const int s = k % kStages;
    const uint32_t parity = (uint32_t)(k / kStages) & 1u;
    const uint8_t* stage = smem + s * Cfg::kStageBytes;
    float2 v[16];
    const bool ok = mbar_wait_bounded(smem_addr(&bars[s]), parity);
    if (ok) {
      load_block<kInBytes>(stage, tid, v);
    } else {
      *abort_flag = 1;
      atomicOr(&g_devstat, (unsigned)KQ_DEVSTAT_WAIT_TIMEOUT);
    }
    __syncthreads();
    if (*abort_flag) {
      // Give the loads still in flight (tiles k .. k + kStages - 1) time to land
      // before the CTA's shared memory goes away, then stop.
      if (tid == 0) {
        for (int kk = k; kk < k + kStages; ++kk) {
          if (blockIdx.x + kk * gridDim.x >= n_tiles) break;
          (void)mbar_wait_bounded(smem_addr(&bars[kk % kStages]), (uint32_t)(kk / kStages) & 1u);
        }
      }
      return;
    }
    if (tid == 0) {
      const int nt = tile + kStages * gridDim.x;
      if (nt < n_tiles) {
        mbar_arrive_expect_tx(smem_addr(&bars[s]), Cfg::kStageBytes);
        tma_load_2d(smem_addr(smem + s * Cfg::kStageBytes), &tmap, 0, nt * kTileBlocks,
                    smem_addr(&bars[s]));
      }
    }

    const int g = tile * kTileBlocks + tid;
    if (g < n_blocks) {
      const float* crow = table + j * kRow;
      if constexpr (kOp == Op::kSqQuant) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 c = *reinterpret_cast<const float4*>(crow + 4 * q);
          v[2 * q + 0] = __fmul2_rn(v[2 * q + 0], make_float2(c.x, c.y));
          v[2 * q + 1] = __fmul2_rn(v[2 * q + 1], make_float2(c.z, c.w));
        }
      } else {
        float4 A[5];
#pragma unroll
        for (int m = 0; m < 5; ++m) A[m] = *reinterpret_cast<const float4*>(crow + 4 * m);
        butterfly32(v, A);
      }
      if constexpr (kOp == Op::kKqTransform) {
        float4* dst = reinterpret_cast<float4*>(y_out + (size_t)g * 32);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          dst[q] = make_float4(v[2 * q].x, v[2 * q].y, v[2 * q + 1].x, v[2 * q + 1].y);
      } else {
        uint4 packed;
        const uint32_t byte = mxfp4_encode32(v, packed);
        *reinterpret_cast<uint4*>(codes + (size_t)g * 16) = packed;
        scales[g] = (uint8_t)byte;
      }
    }
    j += jstep;
    if (j >= nb) j -= nb;
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
cudaError_t g_encode_err = cudaSuccess;

int get_encoder(PFN_cuTensorMapEncodeTiled_v12000* out) {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    g_encode_err = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                                    cudaEnableDefault, &q);
    if (g_encode_err == cudaSuccess && q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) {
    if (g_encode_err != cudaSuccess) return cuda_fail(g_encode_err, "cuTensorMapEncodeTiled lookup");
    return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled not found in the CUDA driver");
  }
  *out = g_encode;
  return KQ_OK;
}

// Tensor map over the flat block view: dim0 = 32 elements, dim1 = n_blocks.
int make_block_tmap(CUtensorMap* tm, const void* x, int x_dtype, int n_blocks) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  if (int st = get_encoder(&enc)) return st;
  const bool bf16 = (x_dtype == KQ_DTYPE_BF16);
  const cuuint64_t dims[2] = {32, (cuuint64_t)n_blocks};
  const cuuint64_t strides[1] = {(cuuint64_t)(bf16 ? 64 : 128)};
  const cuuint32_t box[2] = {32, (cuuint32_t)kTileBlocks};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(tm, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                         2, const_cast<void*>(x), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE,
                         bf16 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return KQ_OK;
}

constexpr int kMaxDevices = 64;

template <int kInBytes, Op kOp>
int launch_stream(const void* x, int x_dtype, int64_t M, int64_t d, const float* coef,
                  uint8_t* codes, uint8_t* scales, float* y, cudaStream_t stream) {
  using Cfg = StreamCfg<kInBytes, kOp>;
  const int nb = (int)(d / 32);
  const int n_blocks = (int)(M * nb);
  auto kern = stream_kernel<kInBytes, kOp>;
  const size_t smem = Cfg::smem_bytes(nb);

  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return cuda_fail(err, "cudaGetDevice");
  // per-device, per-instantiation: raise the dynamic shared memory limit once
  static std::once_flag attr_once[kMaxDevices];
  static cudaError_t attr_err[kMaxDevices];
  if (dev < 0 || dev >= kMaxDevices) return fail(KQ_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::call_once(attr_once[dev], [&] {
    int optin = 0;
    attr_err[dev] = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (attr_err[dev] == cudaSuccess) {
      size_t want = Cfg::smem_bytes(KQ_MAX_D / 32);
      if (want > (size_t)optin) want = (size_t)optin;
      attr_err[dev] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)want);
    }
  });
  if (attr_err[dev] != cudaSuccess) return cuda_fail(attr_err[dev], "cudaFuncSetAttribute");

  int sms = 0;
  if (int st = sm_count(&sms)) return st;
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (err != cudaSuccess) return cuda_fail(err, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
  if (per_sm < 1) return fail(KQ_ERR_UNSUPPORTED, "kernel does not fit on an SM (smem %zu)", smem);

  CUtensorMap tm;
  if (int st = make_block_tmap(&tm, x, x_dtype, n_blocks)) return st;
  const int n_tiles = (n_blocks + kTileBlocks - 1) / kTileBlocks;
  int grid = sms * per_sm;
  if (grid > n_tiles) grid = n_tiles;
  kern<<<grid, kThreads, smem, stream>>>(tm, coef, nb, n_blocks, codes, scales, y);
  return check_launch("stream_kernel launch");
}

template <Op kOp>
int dispatch(const void* x, int x_dtype, int64_t M, int64_t d, const float* coef,
             uint8_t* codes, uint8_t* scales, float* y, void* stream, const char* fn) {
  if (int st = check_shape(M, d, KQ_MAX_D, fn)) return st;
  if (x_dtype != KQ_DTYPE_BF16 && x_dtype != KQ_DTYPE_F32)
    return fail(KQ_ERR_DTYPE, "%s: x_dtype = %d", fn, x_dtype);
  if (M == 0) return KQ_OK;   // nothing to read or write; pointers may be NULL
  if (!x || !coef) return fail(KQ_ERR_INVALID_ARG, "%s: NULL input pointer", fn);
  if (kOp == Op::kKqTransform) {
    if (!y) return fail(KQ_ERR_INVALID_ARG, "%s: NULL output pointer", fn);
  } else if (!codes || !scales) {
    return fail(KQ_ERR_INVALID_ARG, "%s: NULL output pointer", fn);
  }
  if (!aligned(x, 16)) return fail(KQ_ERR_ALIGNMENT, "%s: x must be 16-byte aligned", fn);
  if (!aligned(coef, 4)) return fail(KQ_ERR_ALIGNMENT, "%s: parameters must be 4-byte aligned", fn);
  if (codes && !aligned(codes, 16)) return fail(KQ_ERR_ALIGNMENT, "%s: codes must be 16-byte aligned", fn);
  if (y && !aligned(y, 16)) return fail(KQ_ERR_ALIGNMENT, "%s: y must be 16-byte aligned", fn);
  const cudaStream_t s = as_stream(stream);
  if (x_dtype == KQ_DTYPE_BF16)
    return launch_stream<2, kOp>(x, x_dtype, M, d, coef, codes, scales, y, s);
  return launch_stream<4, kOp>(x, x_dtype, M, d, coef, codes, scales, y, s);
}

}  // namespace
}  // namespace kq

extern "C" {

int kq_quantize(const void* x, int x_dtype, int64_t M, int64_t d, const float* params,
                uint8_t* codes, uint8_t* scales, void* stream) {
  return kq::dispatch<kq::Op::kKqQuant>(x, x_dtype, M, d, params, codes, scales, nullptr, stream,
                                        "kq_quantize");
}

int kq_transform(const void* x, int x_dtype, int64_t M, int64_t d, const float* params, float* y,
                 void* stream) {
  return kq::dispatch<kq::Op::kKqTransform>(x, x_dtype, M, d, params, nullptr, nullptr, y, stream,
                                            "kq_transform");
}

int sq_quantize(const void* x, int x_dtype, int64_t M, int64_t d, const float* inv_s,
                uint8_t* codes, uint8_t* scales, void* stream) {
  return kq::dispatch<kq::Op::kSqQuant>(x, x_dtype, M, d, inv_s, codes, scales, nullptr, stream,
                                        "sq_quantize");
}

int kq_device_status(uint32_t* flags, int clear) {
  if (!flags) return kq::fail(KQ_ERR_INVALID_ARG, "kq_device_status: NULL flags");
  cudaError_t err = cudaDeviceSynchronize();
  if (err != cudaSuccess) return kq::cuda_fail(err, "cudaDeviceSynchronize");
  unsigned int v = 0;
  err = cudaMemcpyFromSymbol(&v, kq::g_devstat, sizeof(v));
  if (err != cudaSuccess) return kq::cuda_fail(err, "cudaMemcpyFromSymbol");
  if (clear) {
    const unsigned int z = 0;
    err = cudaMemcpyToSymbol(kq::g_devstat, &z, sizeof(z));
    if (err != cudaSuccess) return kq::cuda_fail(err, "cudaMemcpyToSymbol");
  }
  *flags = v;
  return KQ_OK;
}

}  // extern "C"
