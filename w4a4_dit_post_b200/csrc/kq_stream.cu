// Streaming kernels of the online quantizer: kq_quantize, kq_transform and
// the SmoothQuant comparison quantizer sq_quantize.
//
// Tiling.  An activation [M][d] is viewed as [M rows][nb blocks][32 elements]
// (rows contiguous, nb = d / 32).  The nb block columns are cut into NC
// column groups of C consecutive blocks (C = the largest divisor of nb not
// above 32) and the rows into row tiles of R rows, R = floor(256 / C).  A
// tile (R x C blocks, at most 16 KiB of bf16) arrives in shared memory by one
// 3-D TMA load (box 32 x C x R, 64-byte swizzle for bf16 rows, 128-byte for
// fp32 rows); the swizzle makes each thread's 16-byte reads of a whole block
// conflict-free.
//
// Column-stationary persistent grid.  The grid is a multiple of NC; CTA b owns
// column group b % NC for its whole life and walks every (G / NC)-th row
// tile.  Its transform coefficients therefore cover only C block columns and
// are built once, in a small shared table.  Thread t owns block column
// t % C and row t / C of every tile: one 32-element block, held as 16
// float2 pairs of adjacent elements.  The first four Kronecker factors pair
// whole float2s, so their shears are packed f32x2 FMAs with a broadcast
// coefficient; the fifth pairs the two halves of each float2 (scalar FMAs).
// One block per thread keeps a thread under 64 registers, so four CTAs (32
// warps) share an SM; in this latency-bound loop the extra warps hide more
// than the packed FMAs of a two-row-per-thread layout (126 registers, 16
// warps per SM) save.  The kernel is also compiled with C fixed at 32 (every
// d that is a multiple of 1024), so that tile height, stage size and the
// thread's block offsets are constants; per tile a thread then only advances
// counters and pointers.
//
// Transform.  Each LU factor A = L U (L = [[1,0],[a,1]], U = [[u,b],[0,1/u]])
// is split as A = S L'' U' with S = diag(u, 1/u), U' = [[1, b/u], [0, 1]] and
// L'' = [[1, 0], [a u^2, 1]].  The diagonal S of one Kronecker position
// commutes with the factors at the other positions, so
//     T = (x)_m A_m = D (x)_m L''_m (x)_m U'_m,   D = (x)_m S_m (diagonal),
// and the block transform is ten shear passes (one FMA per element pair
// each) and one diagonal scaling: 6 flops per element instead of 10.  The
// sizes of the summed terms are unchanged: D |L''| |U'| = |L| |U| entrywise.
//
// Pipeline.  Thread 0 keeps kStages tiles in flight; each stage is guarded by
// an mbarrier (bounded waits).  After copying its block into registers
// a thread joins a CTA barrier, thread 0 reuses the stage for the tile
// kStages ahead, and the transform, the MXFP4 encoding and the stores
// overlap the loads in flight.
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
constexpr int kMaxC = 32;

// kKqCentered: kq_quantize_centered (x - mu formed before the transform).
enum class Op : int { kKqQuant = 0, kKqTransform = 1, kSqQuant = 2, kKqCentered = 3 };

// Tile geometry, computed on the host and passed by value.
struct Geometry {
  int nb;           // blocks per row
  int C;            // blocks per column group
  int NC;           // column groups
  int R;            // rows per tile
  int M;            // rows
  int n_row_tiles;
  int stage_bytes;  // R * C * block bytes, rounded up to 1024
  int sf_tiled;     // 1: scale bytes in the 512-byte blocks kq_gemm_mxfp4 reads
};

// Byte of (row r, scale column s) in the blocked scale layout (512-byte block
// per 128 rows x 4 scale columns; row r's 4 scales at (r % 32) * 16 + (r / 32 % 4) * 4).
__device__ __forceinline__ size_t sf_tiled_offset(int r, int s, int nb) {
  return ((size_t)(r >> 7) * (size_t)(nb >> 2) + (size_t)(s >> 2)) * 512 + (size_t)((r & 31) << 4) +
         (size_t)(((r >> 5) & 3) << 2) + (size_t)(s & 3);
}

template <int kInBytes>
struct InLayout;

template <>
struct InLayout<2> {                     // bf16: 64-byte blocks, 64B swizzle
  static constexpr int kBlockBytes = 64;
  // physical 16-byte chunk of logical chunk q in shared block-row b
  __device__ static int chunk(int b, int q) { return q ^ ((b >> 1) & 3); }
};

template <>
struct InLayout<4> {                     // fp32: 128-byte blocks, 128B swizzle
  static constexpr int kBlockBytes = 128;
  __device__ static int chunk(int b, int q) { return q ^ (b & 7); }
};

// Coefficient table row per block column (floats).  KroQuant: the ten shear
// coefficients, each stored twice (the packed pair of a broadcast operand),
// then the 32 diagonal entries: 52 floats, 13 16-byte units (odd, so 8
// threads on consecutive columns hit distinct bank groups).  SmoothQuant:
// the 32 inverse scales padded to 36 floats (9 units).
template <Op kOp>
struct Table {
  static constexpr int kRowFloats = (kOp == Op::kSqQuant) ? 36 : 52;
};

// CTAs per SM that the register budget is sized for.  bf16 input: four
// (64 registers a thread, 32 warps per SM; four CTAs' shared memory fits).
// kq_transform's fp32 stores need more registers than that: three (85).
// fp32 input: only two CTAs' shared memory fits, so two (128 registers).
template <int kInBytes, Op kOp>
constexpr int min_blocks_per_sm() {
  return kInBytes == 4 ? 2 : (kOp == Op::kKqTransform ? 3 : 4);
}

template <int kInBytes>
struct StageCfg {
  static constexpr int kStages = 2;
};

// Largest divisor of nb that is at most kMaxC.
inline int choose_C(int nb) {
  for (int c = nb < kMaxC ? nb : kMaxC; c > 1; --c)
    if (nb % c == 0) return c;
  return 1;
}

template <int kInBytes>
inline Geometry make_geometry(int64_t M, int nb) {
  Geometry g;
  g.nb = nb;
  g.C = choose_C(nb);
  g.NC = nb / g.C;
  int R = kThreads / g.C;
  if (R > 256) R = 256;                  // TMA box dimension limit
  g.R = R;
  g.M = (int)M;
  g.n_row_tiles = (int)((M + R - 1) / R);
  const int raw = R * g.C * InLayout<kInBytes>::kBlockBytes;
  g.stage_bytes = (raw + 1023) & ~1023;
  return g;
}

// Stage size of a tile when the column-group width kC is fixed at compile time
// (the same formula as make_geometry's: R = kThreads / C rows).
template <int kInBytes, int kC>
struct FixedStageBytes {
  static constexpr int value =
      ((kThreads / kC) * kC * InLayout<kInBytes>::kBlockBytes + 1023) & ~1023;
};

template <int kInBytes, Op kOp>
inline size_t smem_bytes(const Geometry& g) {
  // + staging for the raw coefficients: C * 32 floats
  return 1024 /* base alignment */ + (size_t)StageCfg<kInBytes>::kStages * g.stage_bytes + 128 +
         (size_t)g.C * (Table<kOp>::kRowFloats + 32) * sizeof(float);
}

// One block (row r of block column c of a tile) from a stage: v[k] holds
// elements (2k, 2k+1).
template <int kInBytes>
__device__ __forceinline__ void load_row(const uint8_t* stage, int C, int r, int c, float2 (&v)[16]) {
  using L = InLayout<kInBytes>;
  const int b = r * C + c;
  const uint8_t* p = stage + b * L::kBlockBytes;
  if constexpr (kInBytes == 2) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 w = *reinterpret_cast<const uint4*>(p + (L::chunk(b, q) << 4));
      v[4 * q + 0] = bf16x2_to_float2(w.x);
      v[4 * q + 1] = bf16x2_to_float2(w.y);
      v[4 * q + 2] = bf16x2_to_float2(w.z);
      v[4 * q + 3] = bf16x2_to_float2(w.w);
    }
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 w = *reinterpret_cast<const float4*>(p + (L::chunk(b, q) << 4));
      v[2 * q] = make_float2(w.x, w.y);
      v[2 * q + 1] = make_float2(w.z, w.w);
    }
  }
}

// KroQuant transform of one block from its coefficient row.  Row layout:
// floats [4m .. 4m+3] = (b_m/u_m, b_m/u_m, a_m u_m^2, a_m u_m^2) for m = 0..4,
// then [20 + i] = D_i for i = 0..31.  Factor m acts on element-index bit
// 4 - m, i.e. on bit 3 - m of the pair index k for m < 4 (whole float2s,
// packed FMA) and inside each float2 for m = 4.
__device__ __forceinline__ void kq_transform_row(float2 (&v)[16], const float* row) {
  const float4* r4 = reinterpret_cast<const float4*>(row);
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int h = 1 << (3 - m);
    const float4 sh = r4[m];
    const float2 beta = make_float2(sh.x, sh.y), gamma = make_float2(sh.z, sh.w);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      if (k & h) continue;
      v[k] = __ffma2_rn(beta, v[k + h], v[k]);        // U':  lo += (b/u) hi
      v[k + h] = __ffma2_rn(gamma, v[k], v[k + h]);   // L'':  hi += (a u^2) lo
    }
  }
  {
    const float4 sh = r4[4];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      v[k].x = __fmaf_rn(sh.x, v[k].y, v[k].x);
      v[k].y = __fmaf_rn(sh.z, v[k].x, v[k].y);
    }
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 dd = r4[5 + q];            // D_4q .. D_4q+3
    v[2 * q] = __fmul2_rn(v[2 * q], make_float2(dd.x, dd.y));
    v[2 * q + 1] = __fmul2_rn(v[2 * q + 1], make_float2(dd.z, dd.w));
  }
}

__device__ __forceinline__ void sq_transform_row(float2 (&v)[16], const float* row) {
  const float4* r4 = reinterpret_cast<const float4*>(row);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 s = r4[q];
    v[2 * q] = __fmul2_rn(v[2 * q], make_float2(s.x, s.y));
    v[2 * q + 1] = __fmul2_rn(v[2 * q + 1], make_float2(s.z, s.w));
  }
}

// Transform of one block (row r, block column jc) and its output: the
// transformed values (kq_transform), or the E2M1 codes and E8M0 scale byte.
// cdst, sdst and ydst point at the block in codes, scales and y.
template <Op kOp>
__device__ __forceinline__ void quantize_row(float2 (&v)[16], const float* crow, const Geometry& geo,
                                             int r, int jc, uint8_t* cdst, uint8_t* sdst, float* ydst,
                                             uint8_t* __restrict__ scales) {
  if constexpr (kOp == Op::kSqQuant) {
    sq_transform_row(v, crow);
  } else {
    kq_transform_row(v, crow);
  }
  if constexpr (kOp == Op::kKqTransform) {
    float4* d0 = reinterpret_cast<float4*>(ydst);
#pragma unroll
    for (int q = 0; q < 8; ++q) d0[q] = make_float4(v[2 * q].x, v[2 * q].y, v[2 * q + 1].x, v[2 * q + 1].y);
  } else {
    uint4 out;
    const uint32_t e = mxfp4_encode32(v, out);
    *reinterpret_cast<uint4*>(cdst) = out;
    if (geo.sf_tiled) {
      scales[sf_tiled_offset(r, jc, geo.nb)] = (uint8_t)e;
    } else {
      *sdst = (uint8_t)e;
    }
  }
}

// kC: the column-group width when it is fixed at compile time (32, every
// d that is a multiple of 1024), else 0 and the width comes from geo.
template <int kInBytes, Op kOp, int kC>
__global__ void __launch_bounds__(kThreads, (min_blocks_per_sm<kInBytes, kOp>()))
stream_kernel(const __grid_constant__ CUtensorMap tmap, const float* __restrict__ coef_src,
              const Geometry geo, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
              float* __restrict__ y_out, const float* __restrict__ mu) {
  constexpr int kStages = StageCfg<kInBytes>::kStages;
  constexpr int kRow = Table<kOp>::kRowFloats;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  // with a fixed group width the tile geometry is a compile-time constant
  const int stage_bytes = kC ? FixedStageBytes<kInBytes, (kC ? kC : 32)>::value : geo.stage_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * stage_bytes);
  float* table = reinterpret_cast<float*>(smem + kStages * stage_bytes + 128);

  const int tid = threadIdx.x;
  __builtin_assume(tid < kThreads);
  const int C = kC ? kC : geo.C, R = kC ? (kThreads / (kC ? kC : 1)) : geo.R;
  const int col_group = blockIdx.x % geo.NC;
  const int row_step = gridDim.x / geo.NC;      // CTAs sharing this column group
  const int rt_first = blockIdx.x / geo.NC;
  const int j0 = col_group * C;                 // first block column of the group
  const uint32_t tile_tx = (uint32_t)(R * C * InLayout<kInBytes>::kBlockBytes);

  // Programmatic dependent launch: let the next kernel in the stream begin
  // launching now, and touch no global memory before the previous kernel in
  // the stream has completed (griddepcontrol.wait returns at once when this
  // launch has no programmatic predecessor).
  //
  // Before that wait the CTA only asks for its first tiles and its
  // coefficients to be brought into L2.  A prefetch changes no memory and L2
  // is where every write of the previous kernel lands, so the loads after the
  // wait still see that kernel's results; they just find them on chip.  This
  // overlaps the start of this launch with the tail of the previous one.
  pdl_launch_dependents();
  if (tid == 0) {
    tma_prefetch_desc(&tmap);
#pragma unroll
    for (int s = 0; s < kStages; ++s) mbar_init(smem_addr(&bars[s]), 1);
    mbar_init_fence();
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
      const int rt = rt_first + s * row_step;
      if (rt < geo.n_row_tiles) tma_prefetch_l2_3d(&tmap, 0, j0, rt * R);
    }
  }
  {
    constexpr int kCoefPerBlock = (kOp == Op::kSqQuant) ? 32 : 15;
    const char* cbase = reinterpret_cast<const char*>(coef_src + kCoefPerBlock * j0);
    const int cbytes = C * kCoefPerBlock * 4;
    const int first = tid * 128 - (int)(reinterpret_cast<uintptr_t>(cbase) & 127);
    if (tid < 32 && first < cbytes) prefetch_l2(cbase + (first > 0 ? first : 0));
  }
  pdl_wait_predecessor();
  __syncthreads();
  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
      const int rt = rt_first + s * row_step;
      if (rt < geo.n_row_tiles) {
        mbar_arrive_expect_tx(smem_addr(&bars[s]), tile_tx);
        tma_load_3d(smem_addr(smem + s * stage_bytes), &tmap, 0, j0, rt * R, smem_addr(&bars[s]));
      }
    }
  }

  // Coefficients of this CTA's C block columns, overlapping the first loads.
  // The raw parameters are staged with asynchronous copies (all in flight at
  // once: one memory round trip), then turned into table rows from shared
  // memory only.
  if constexpr (kOp == Op::kSqQuant) {
    float* stage_in = table + C * kRow;                 // C * 32 inverse scales
    for (int i = tid; i < C * 32; i += kThreads) cp_async_4(smem_addr(stage_in + i), coef_src + 32 * j0 + i);
    cp_async_wait_all();
    __syncthreads();
    for (int i = tid; i < C * 32; i += kThreads) {
      const float sv = stage_in[i];
      table[(i >> 5) * kRow + (i & 31)] = sv;
    }
  } else {
    float* prm = table + C * kRow;                      // C * 15 parameters
    float* uu = prm + C * 16;                           // C * 10: (u_m, 1/u_m)
    for (int i = tid; i < C * 15; i += kThreads) cp_async_4(smem_addr(prm + i), coef_src + 15 * j0 + i);
    cp_async_wait_all();
    __syncthreads();
    // thread (c, m): the two shears of factor m and (u, 1/u)
    for (int i = tid; i < C * 5; i += kThreads) {
      const int cc = i / 5, m = i - 5 * cc;
      const float a = prm[15 * cc + 3 * m], b = prm[15 * cc + 3 * m + 1], u = prm[15 * cc + 3 * m + 2];
      if (lu_params_bad(a, b, u)) atomicOr(&g_devstat, (unsigned)KQ_DEVSTAT_BAD_PARAMS);
      const float beta = b / u, gamma = __fmul_rn(__fmul_rn(a, u), u);
      *reinterpret_cast<float4*>(table + cc * kRow + 4 * m) = make_float4(beta, beta, gamma, gamma);
      uu[10 * cc + 2 * m] = u;
      uu[10 * cc + 2 * m + 1] = 1.0f / u;
    }
    __syncthreads();
    // thread (c, e): D_e = prod_m (bit (4 - m) of e ? 1/u_m : u_m)
    for (int i = tid; i < C * 32; i += kThreads) {
      const int cc = i >> 5, e = i & 31;
      float dval = 1.0f;
#pragma unroll
      for (int m = 0; m < 5; ++m) dval = __fmul_rn(dval, uu[10 * cc + 2 * m + ((e >> (4 - m)) & 1)]);
      table[cc * kRow + 20 + e] = dval;
    }
  }
  __syncthreads();

  const int c = tid % C, rr = tid / C;
  const bool active = rr < R;
  const float* crow = table + c * kRow;
  const int nb = geo.nb;

  // Tiles walk the stages in order; the barrier phase flips once per round of
  // kStages tiles (a counter and a flag instead of a division per tile).
  int rt = rt_first;
  uint32_t parity = 0;
  // This thread's row (unsigned: the host refuses M >= 2^30, so it stays
  // below 2^31 + 2^9 even one step past the last tile) and the addresses of
  // its output block, advanced by a constant per tile.  The addresses are
  // kept as integers: after the last tile they step past the buffers, and
  // unsigned arithmetic makes that well defined; they are only dereferenced
  // for rows below M.
  uint32_t r0 = (uint32_t)(rt_first * R + rr);
  const uint32_t r_step = (uint32_t)(row_step * R);
  const size_t g_first = (size_t)r0 * nb + j0 + c, g_step = (size_t)r_step * nb;
  constexpr bool kCodes = kOp != Op::kKqTransform;   // the other output is NULL
  uintptr_t cdst = kCodes ? reinterpret_cast<uintptr_t>(codes) + g_first * 16 : 0;
  uintptr_t sdst = kCodes ? reinterpret_cast<uintptr_t>(scales) + g_first : 0;
  uintptr_t ydst = kCodes ? 0 : reinterpret_cast<uintptr_t>(y_out) + g_first * 128;
  for (;;) {
#pragma unroll 1
    for (int s = 0; s < kStages; ++s, rt += row_step, r0 += r_step) {
      if (rt >= geo.n_row_tiles) return;
      float2 v[16];
      // centring variant: this row's offset (read before the wait, so the
      // load overlaps it)
      float2 neg_mu = make_float2(0.0f, 0.0f);
      if (kOp == Op::kKqCentered && active && r0 < (uint32_t)geo.M) neg_mu = make_float2(-mu[r0], -mu[r0]);
      const bool ok = mbar_wait_bounded(smem_addr(&bars[s]), parity);
      if (ok) {
        if (active) {
          load_row<kInBytes>(smem + s * stage_bytes, C, rr, c, v);
          if constexpr (kOp == Op::kKqCentered) {
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = __fadd2_rn(v[i], neg_mu);
          }
        }
      } else {
        atomicOr(&g_devstat, (unsigned)KQ_DEVSTAT_WAIT_TIMEOUT);
      }
      // one barrier per tile, which also tells every thread whether any wait ran out
      if (__syncthreads_or(!ok)) {
        // let the loads still in flight land before shared memory goes away:
        // this tile's and the next kStages - 1, in the following stages
        if (tid == 0) {
          for (int i = 0; i < kStages; ++i) {
            if (rt + i * row_step >= geo.n_row_tiles) break;
            const int si = (s + i) % kStages;
            const uint32_t pi = parity ^ (uint32_t)((s + i) / kStages);
            (void)mbar_wait_bounded(smem_addr(&bars[si]), pi & 1u);
          }
        }
        return;
      }
      if (tid == 0) {
        const int nrt = rt + kStages * row_step;
        if (nrt < geo.n_row_tiles) {
          mbar_arrive_expect_tx(smem_addr(&bars[s]), tile_tx);
          tma_load_3d(smem_addr(smem + s * stage_bytes), &tmap, 0, j0, nrt * R, smem_addr(&bars[s]));
        }
      }
      if (active && r0 < (uint32_t)geo.M)
        quantize_row<kOp>(v, crow, geo, (int)r0, j0 + c, reinterpret_cast<uint8_t*>(cdst),
                          reinterpret_cast<uint8_t*>(sdst), reinterpret_cast<float*>(ydst), scales);
      if constexpr (kCodes) {
        cdst += g_step * 16;
        sdst += g_step;
      } else {
        ydst += g_step * 128;
      }
    }
    parity ^= 1u;
  }
}

// Failure-detection self-test: one thread waits on a barrier that nothing
// arrives on, through the same bounded wait the streaming kernels use.  The
// wait runs out after limit_ns, sets the status bit and the kernel returns.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(smem_addr(&bar), 1);
  mbar_init_fence();
  if (!mbar_wait_bounded(smem_addr(&bar), 0u, limit_ns))
    atomicOr(&g_devstat, (unsigned)KQ_DEVSTAT_WAIT_TIMEOUT);
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

// Tensor map over [M][nb][32]: box = 32 elements x C blocks x R rows.
template <int kInBytes>
int make_tile_tmap(CUtensorMap* tm, const void* x, const Geometry& g) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  if (int st = get_encoder(&enc)) return st;
  const cuuint64_t dims[3] = {32, (cuuint64_t)g.nb, (cuuint64_t)g.M};
  const cuuint64_t strides[2] = {(cuuint64_t)(32 * kInBytes), (cuuint64_t)g.nb * 32 * kInBytes};
  const cuuint32_t box[3] = {32, (cuuint32_t)g.C, (cuuint32_t)g.R};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r =
      enc(tm, kInBytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
          const_cast<void*>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          kInBytes == 2 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return KQ_OK;
}

constexpr int kMaxDevices = 64;

template <int kInBytes, Op kOp>
int launch_stream(const void* x, int64_t M, int64_t d, const float* coef, uint8_t* codes,
                  uint8_t* scales, float* y, cudaStream_t stream, bool sf_tiled, const float* mu) {
  const int nb = (int)(d / 32);
  Geometry geo = make_geometry<kInBytes>(M, nb);
  geo.sf_tiled = sf_tiled ? 1 : 0;
  auto kern = geo.C == 32 ? stream_kernel<kInBytes, kOp, 32> : stream_kernel<kInBytes, kOp, 0>;
  const size_t smem = smem_bytes<kInBytes, kOp>(geo);
  if (geo.C == 32 && geo.stage_bytes != FixedStageBytes<kInBytes, 32>::value)
    return fail(KQ_ERR_UNSUPPORTED, "internal: tile geometry of the fixed-width kernel disagrees with the host");

  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return cuda_fail(err, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(KQ_ERR_UNSUPPORTED, "device ordinal %d", dev);
  // per device and instantiation (both group-width variants): allow the
  // largest dynamic shared memory once
  static std::once_flag attr_once[kMaxDevices];
  static cudaError_t attr_err[kMaxDevices];
  std::call_once(attr_once[dev], [&] {
    int optin = 0;
    attr_err[dev] = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (attr_err[dev] == cudaSuccess)
      attr_err[dev] = cudaFuncSetAttribute(stream_kernel<kInBytes, kOp, 32>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (attr_err[dev] == cudaSuccess)
      attr_err[dev] = cudaFuncSetAttribute(stream_kernel<kInBytes, kOp, 0>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  });
  if (attr_err[dev] != cudaSuccess) return cuda_fail(attr_err[dev], "cudaFuncSetAttribute");

  int sms = 0;
  if (int st = sm_count(&sms)) return st;
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (err != cudaSuccess) return cuda_fail(err, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
  if (per_sm < 1) return fail(KQ_ERR_UNSUPPORTED, "kernel does not fit on an SM (smem %zu)", smem);

  CUtensorMap tm;
  if (int st = make_tile_tmap<kInBytes>(&tm, x, geo)) return st;
  // a whole number of CTAs per column group, no more than there are row tiles
  const int64_t slots = (int64_t)sms * per_sm;
  int64_t per_group = slots / geo.NC;
  if (per_group < 1) per_group = 1;
  if (per_group > geo.n_row_tiles) per_group = geo.n_row_tiles;
  const int64_t grid = per_group * geo.NC;
  // launched with programmatic stream serialization (see the kernel's prologue)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, kern, tm, coef, geo, codes, scales, y, mu);
  if (err != cudaSuccess) return cuda_fail(err, "stream_kernel launch");
  return check_launch("stream_kernel launch");
}

template <Op kOp>
int dispatch(const void* x, int x_dtype, int64_t M, int64_t d, const float* coef,
             uint8_t* codes, uint8_t* scales, float* y, void* stream, const char* fn,
             bool sf_tiled = false, const float* mu = nullptr, bool need_mu = false) {
  if (int st = check_shape(M, d, KQ_MAX_D, fn)) return st;
  if (M >= ((int64_t)1 << 30))
    return fail(KQ_ERR_UNSUPPORTED, "%s: M = %lld rows exceeds the limit 2^30 - 1", fn, (long long)M);
  if (sf_tiled && d % 128 != 0)
    return fail(KQ_ERR_INVALID_ARG, "%s: d must be a multiple of 128 (d = %lld)", fn, (long long)d);
  if (x_dtype != KQ_DTYPE_BF16 && x_dtype != KQ_DTYPE_F32)
    return fail(KQ_ERR_DTYPE, "%s: x_dtype = %d", fn, x_dtype);
  if (M == 0) return KQ_OK;   // nothing to read or write; pointers may be NULL
  if (!x || !coef) return fail(KQ_ERR_INVALID_ARG, "%s: NULL input pointer", fn);
  if (kOp == Op::kKqTransform) {
    if (!y) return fail(KQ_ERR_INVALID_ARG, "%s: NULL output pointer", fn);
  } else if (!codes || !scales) {
    return fail(KQ_ERR_INVALID_ARG, "%s: NULL output pointer", fn);
  }
  if (need_mu && !mu) return fail(KQ_ERR_INVALID_ARG, "%s: NULL mu", fn);
  if (mu && !aligned(mu, 4)) return fail(KQ_ERR_ALIGNMENT, "%s: mu must be 4-byte aligned", fn);
  if (!aligned(x, 16)) return fail(KQ_ERR_ALIGNMENT, "%s: x must be 16-byte aligned", fn);
  if (!aligned(coef, 4)) return fail(KQ_ERR_ALIGNMENT, "%s: parameters must be 4-byte aligned", fn);
  if (codes && !aligned(codes, 16)) return fail(KQ_ERR_ALIGNMENT, "%s: codes must be 16-byte aligned", fn);
  if (y && !aligned(y, 16)) return fail(KQ_ERR_ALIGNMENT, "%s: y must be 16-byte aligned", fn);
  const cudaStream_t s = as_stream(stream);
  if (x_dtype == KQ_DTYPE_BF16) return launch_stream<2, kOp>(x, M, d, coef, codes, scales, y, s, sf_tiled, mu);
  return launch_stream<4, kOp>(x, M, d, coef, codes, scales, y, s, sf_tiled, mu);
}

}  // namespace
}  // namespace kq

namespace kq {

int device_status_address(unsigned int** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return cuda_fail(err, "cudaGetDevice");
  static std::mutex mu;
  static unsigned int* addr[64] = {nullptr};
  if (dev < 0 || dev >= 64) return fail(KQ_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_devstat);
    if (err != cudaSuccess) return cuda_fail(err, "cudaGetSymbolAddress(status word)");
    addr[dev] = static_cast<unsigned int*>(p);
  }
  *out = addr[dev];
  return KQ_OK;
}

}  // namespace kq

extern "C" {

int kq_quantize(const void* x, int x_dtype, int64_t M, int64_t d, const float* params,
                uint8_t* codes, uint8_t* scales, void* stream) {
  return kq::dispatch<kq::Op::kKqQuant>(x, x_dtype, M, d, params, codes, scales, nullptr, stream,
                                        "kq_quantize");
}

int kq_quantize_centered(const void* x, int x_dtype, int64_t M, int64_t d, const float* params,
                         const float* mu, uint8_t* codes, uint8_t* scales, void* stream) {
  return kq::dispatch<kq::Op::kKqCentered>(x, x_dtype, M, d, params, codes, scales, nullptr, stream,
                                           "kq_quantize_centered", false, mu, true);
}

int kq_quantize_sf_tiled(const void* x, int x_dtype, int64_t M, int64_t d, const float* params,
                         uint8_t* codes, uint8_t* scales_tiled, void* stream) {
  return kq::dispatch<kq::Op::kKqQuant>(x, x_dtype, M, d, params, codes, scales_tiled, nullptr,
                                        stream, "kq_quantize_sf_tiled", true);
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

int kq_selftest_bounded_wait(uint32_t limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000)
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_selftest_bounded_wait: limit_us = %u not in [1, 1e6]",
                    limit_us);
  kq::selftest_wait_kernel<<<1, 32, 0, kq::as_stream(stream)>>>((uint64_t)limit_us * 1000ull);
  return kq::check_launch("selftest_wait_kernel launch");
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
