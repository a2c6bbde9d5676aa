// Support kernels: the dense blocks of the transform (kq_expand_params), the
// inverse folded into the weights (kq_fold_weights), the folded weights
// quantised to MXFP4 (kq_quantize_weights) and MXFP4 decoding (kq_dequant).
// None of them is on the per-step path; they are memory-bound kernels.
#include <cuda_runtime.h>

#include "kq.h"
#include "kq_device.cuh"
#include "kq_host.h"

namespace kq {
namespace {

constexpr int kAuxThreads = 256;

// T[j][i][k] = prod_m A_jm[bit(i, 4-m)][bit(k, 4-m)], one thread per entry.
__global__ void __launch_bounds__(kAuxThreads)
expand_kernel(const float* __restrict__ params, int nb, float* __restrict__ T, unsigned int* devstat) {
  const int total = nb * 1024;
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += gridDim.x * blockDim.x) {
    const int j = idx >> 10, i = (idx >> 5) & 31, k = idx & 31;
    const float* p = params + 15 * j;
    if ((idx & 1023) < 5 && lu_params_bad(p[3 * (idx & 1023)], p[3 * (idx & 1023) + 1], p[3 * (idx & 1023) + 2]))
      atomicOr(devstat, (unsigned)KQ_DEVSTAT_BAD_PARAMS);
    float v = 1.0f;
#pragma unroll
    for (int m = 0; m < 5; ++m) {
      const float4 A = lu_factor(p[3 * m], p[3 * m + 1], p[3 * m + 2]);
      const int bi = (i >> (4 - m)) & 1, bk = (k >> (4 - m)) & 1;
      const float e = bi ? (bk ? A.w : A.z) : (bk ? A.y : A.x);
      v = __fmul_rn(v, e);
    }
    T[idx] = v;
  }
}

// The fold with coalesced traffic: a warp takes 32 consecutive blocks (4 KiB
// of W), reads them with 16-byte loads into shared memory (chunk c of block b
// at c ^ (b % 8): conflict-free both ways), each lane folds its own block and
// puts it back in the same slots, and the warp writes the 4 KiB with 16-byte
// stores.  The warp has read its whole piece before it writes any of it, and
// warps own disjoint pieces, so in-place use stays safe.  kCS (nb a multiple
// of 32): the warp keeps one 32-block column group and walks the rows, so
// each lane builds its five transposed inverse factors once; otherwise every
// block loads its own parameters.
template <bool kCS>
__global__ void __launch_bounds__(kAuxThreads)
fold_coalesced_kernel(const float* W, const float* __restrict__ params, int N, int nb, int n_blocks,
                      float* W_out, unsigned int* devstat) {
  __shared__ float4 stage[kAuxThreads / 32][32 * 8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float4* st = stage[warp];
  const int warps_total = gridDim.x * (blockDim.x >> 5);
  const int wglob = blockIdx.x * (blockDim.x >> 5) + warp;
  const int n_cg = nb / 32;
  float4 B[5];
  if constexpr (kCS) {
    // warps past the last whole round of column groups would repeat pieces
    // of the warps below them (harmful in place): they leave
    if (wglob >= (warps_total / n_cg) * n_cg) return;      // warp-uniform
    const int j = (wglob % n_cg) * 32 + lane;
    const float* p = params + 15 * j;
    bool bad = false;
#pragma unroll
    for (int m = 0; m < 5; ++m) {
      bad |= lu_params_bad(p[3 * m], p[3 * m + 1], p[3 * m + 2]);
      B[m] = lu_factor_inv_t(p[3 * m], p[3 * m + 1], p[3 * m + 2]);
    }
    if (bad && wglob < n_cg) atomicOr(devstat, (unsigned)KQ_DEVSTAT_BAD_PARAMS);
  }
  // piece u: kCS -> row u / n_cg, column group u % n_cg (the step keeps the
  // group); otherwise blocks 32 u .. 32 u + 31 of the flattened weight
  const int n_pieces = kCS ? N * n_cg : (n_blocks + 31) / 32;
  const int step = kCS ? (warps_total / n_cg) * n_cg : warps_total;
  for (int u = wglob; u < n_pieces; u += step) {
    const size_t g0 = kCS ? (size_t)(u / n_cg) * nb + (size_t)(u % n_cg) * 32 : (size_t)u * 32;
    const int nblk = kCS ? 32 : (n_blocks - (int)g0 < 32 ? n_blocks - (int)g0 : 32);
    const float4* src = reinterpret_cast<const float4*>(W + g0 * 32);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int L = lane + 32 * i;            // 16-byte chunk of the warp's 4 KiB
      const int b = L >> 3, c = L & 7;
      if (kCS || L < nblk * 8) st[b * 8 + (c ^ (b & 7))] = src[L];
    }
    __syncwarp();
    if (kCS || lane < nblk) {
      if constexpr (!kCS) {
        const int g = (int)g0 + lane;
        const float* p = params + 15 * (g % nb);
        bool bad = false;
#pragma unroll
        for (int m = 0; m < 5; ++m) {
          bad |= lu_params_bad(p[3 * m], p[3 * m + 1], p[3 * m + 2]);
          B[m] = lu_factor_inv_t(p[3 * m], p[3 * m + 1], p[3 * m + 2]);
        }
        if (bad && g < nb) atomicOr(devstat, (unsigned)KQ_DEVSTAT_BAD_PARAMS);
      }
      float2 v[16];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 t = st[lane * 8 + (q ^ (lane & 7))];
        v[2 * q] = make_float2(t.x, t.y);
        v[2 * q + 1] = make_float2(t.z, t.w);
      }
      butterfly32(v, B);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        st[lane * 8 + (q ^ (lane & 7))] = make_float4(v[2 * q].x, v[2 * q].y, v[2 * q + 1].x, v[2 * q + 1].y);
    }
    __syncwarp();
    float4* dst = reinterpret_cast<float4*>(W_out + g0 * 32);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int L = lane + 32 * i;
      const int b = L >> 3, c = L & 7;
      if (kCS || L < nblk * 8) dst[L] = st[b * 8 + (c ^ (b & 7))];
    }
    __syncwarp();
  }
}

// Weight side: one thread per (weight row, block): the folded block
// w T_j^{-1} (the same butterfly as fold_coalesced_kernel) encoded to MXFP4 in
// registers; the folded weights are never written.  A warp takes 32
// consecutive blocks (4 KiB of W): it reads them with coalesced 16-byte loads
// into shared memory (16-byte chunk c of block b stored at chunk c ^ (b % 8),
// so both the writes and the per-block reads are free of bank conflicts),
// then every lane works on its own block; the codes of the 32 blocks leave
// as 512 contiguous bytes, the scales as 32.
__global__ void __launch_bounds__(kAuxThreads)
fold_quant_kernel(const float* __restrict__ W, const float* __restrict__ params, int nb,
                  int n_blocks, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                  unsigned int* devstat) {
  __shared__ float4 stage[kAuxThreads / 32][32 * 8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float4* st = stage[warp];
  const int n_groups = (n_blocks + 31) / 32;
  const int warps_total = gridDim.x * (blockDim.x >> 5);
  for (int wg = blockIdx.x * (blockDim.x >> 5) + warp; wg < n_groups; wg += warps_total) {
    const int g0 = wg * 32;
    const int nblk = n_blocks - g0 < 32 ? n_blocks - g0 : 32;
    const float4* src = reinterpret_cast<const float4*>(W + (size_t)g0 * 32);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int L = lane + 32 * i;            // 16-byte chunk of the warp's 4 KiB
      if (L < nblk * 8) {
        const int b = L >> 3, c = L & 7;
        st[b * 8 + (c ^ (b & 7))] = src[L];
      }
    }
    __syncwarp();
    if (lane < nblk) {
      const int g = g0 + lane;
      const int j = g % nb;
      const float* p = params + 15 * j;
      float4 B[5];
      bool bad = false;
#pragma unroll
      for (int m = 0; m < 5; ++m) {
        bad |= lu_params_bad(p[3 * m], p[3 * m + 1], p[3 * m + 2]);
        B[m] = lu_factor_inv_t(p[3 * m], p[3 * m + 1], p[3 * m + 2]);
      }
      if (bad && g < nb) atomicOr(devstat, (unsigned)KQ_DEVSTAT_BAD_PARAMS);
      float2 v[16];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 t = st[lane * 8 + (q ^ (lane & 7))];
        v[2 * q] = make_float2(t.x, t.y);
        v[2 * q + 1] = make_float2(t.z, t.w);
      }
      butterfly32(v, B);
      uint4 packed;
      const uint32_t byte = mxfp4_encode32(v, packed);
      *reinterpret_cast<uint4*>(codes + (size_t)g * 16) = packed;
      scales[g] = (uint8_t)byte;
    }
    __syncwarp();
  }
}

// The same, column-stationary, when nb is a multiple of 32: warp w keeps the
// 32-block column group w % n_cg of the weight rows w / n_cg, w / n_cg + rstep,
// ..., so each lane keeps one block column and builds its five transposed
// inverse factors once, instead of loading the 15 parameters and dividing for
// every block.  Loads, shared-memory transpose and stores as fold_quant_kernel.
__global__ void __launch_bounds__(kAuxThreads)
fold_quant_cs_kernel(const float* __restrict__ W, const float* __restrict__ params, int N, int nb,
                     int rstep, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                     unsigned int* devstat) {
  __shared__ float4 stage[kAuxThreads / 32][32 * 8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float4* st = stage[warp];
  const int n_cg = nb / 32;
  const int wglob = blockIdx.x * (blockDim.x >> 5) + warp;
  if (wglob >= rstep * n_cg) return;          // warp-uniform
  const int cg = wglob % n_cg;
  const int j = cg * 32 + lane;               // this lane's block column
  const float* p = params + 15 * j;
  float4 B[5];
  bool bad = false;
#pragma unroll
  for (int m = 0; m < 5; ++m) {
    bad |= lu_params_bad(p[3 * m], p[3 * m + 1], p[3 * m + 2]);
    B[m] = lu_factor_inv_t(p[3 * m], p[3 * m + 1], p[3 * m + 2]);
  }
  if (bad && wglob < n_cg) atomicOr(devstat, (unsigned)KQ_DEVSTAT_BAD_PARAMS);
  for (int r = wglob / n_cg; r < N; r += rstep) {
    const size_t g0 = (size_t)r * nb + (size_t)cg * 32;
    const float4* src = reinterpret_cast<const float4*>(W + g0 * 32);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int L = lane + 32 * i;            // 16-byte chunk of the warp's 4 KiB
      const int b = L >> 3, c = L & 7;
      st[b * 8 + (c ^ (b & 7))] = src[L];
    }
    __syncwarp();
    float2 v[16];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 t = st[lane * 8 + (q ^ (lane & 7))];
      v[2 * q] = make_float2(t.x, t.y);
      v[2 * q + 1] = make_float2(t.z, t.w);
    }
    __syncwarp();
    butterfly32(v, B);
    uint4 packed;
    const uint32_t byte = mxfp4_encode32(v, packed);
    *reinterpret_cast<uint4*>(codes + (g0 + lane) * 16) = packed;
    scales[g0 + lane] = (uint8_t)byte;
  }
}

// out[r] = scale * sum of row r (bf16 or fp32 input, fp32 accumulation):
// one warp per row, 16-byte loads.
__global__ void __launch_bounds__(kAuxThreads)
row_sum_kernel(const void* __restrict__ x, int bf16, int M, int d, float scale, float* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (blockDim.x >> 5);
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < M; r += warps) {
    float acc = 0.0f;
    if (bf16) {
      const uint4* row = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + (size_t)r * d);
      for (int i = lane; i < d / 8; i += 32) {
        const uint4 w = row[i];
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          acc += __uint_as_float(ws[e] << 16) + __uint_as_float(ws[e] & 0xffff0000u);
      }
    } else {
      const float4* row = reinterpret_cast<const float4*>(static_cast<const float*>(x) + (size_t)r * d);
      for (int i = lane; i < d / 4; i += 32) {
        const float4 f = row[i];
        acc += (f.x + f.y) + (f.z + f.w);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) out[r] = acc * scale;
  }
}

// E2M1 magnitude of a 3-bit code: 0, 0.5, 1, 1.5, 2, 3, 4, 6.
__device__ __forceinline__ float e2m1_mag(uint32_t c) {
  // exponent field e = c >> 1, mantissa bit m = c & 1:
  // e == 0: m * 0.5 (subnormal); else 2^(e-1) * (1 + m / 2).
  const uint32_t e = c >> 1, m = c & 1u;
  if (e == 0) return m ? 0.5f : 0.0f;
  return __uint_as_float((126u + e) << 23) * (m ? 1.5f : 1.0f);
}

// One thread per block: 16 code bytes + 1 scale byte -> 32 fp32 values.
__global__ void __launch_bounds__(kAuxThreads)
dequant_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales, int n_blocks,
               float* __restrict__ out) {
  for (int g = blockIdx.x * blockDim.x + threadIdx.x; g < n_blocks; g += gridDim.x * blockDim.x) {
    const uint4 c = *reinterpret_cast<const uint4*>(codes + (size_t)g * 16);
    const uint32_t byte = scales[g];
    // 2^(byte - 127): byte 0 is the subnormal 2^-127, 0xFF is NaN
    const uint32_t sbits = byte == 255u ? 0x7fc00000u : (byte == 0u ? 0x00400000u : byte << 23);
    const float s = __uint_as_float(sbits);
    const uint32_t words[4] = {c.x, c.y, c.z, c.w};
    float4* dst = reinterpret_cast<float4*>(out + (size_t)g * 32);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      float f[8];
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const uint32_t nib = (words[w] >> (4 * n)) & 0xFu;
        const float mag = __fmul_rn(e2m1_mag(nib & 7u), s);
        f[n] = (nib & 8u) ? -mag : mag;
      }
      dst[2 * w] = make_float4(f[0], f[1], f[2], f[3]);
      dst[2 * w + 1] = make_float4(f[4], f[5], f[6], f[7]);
    }
  }
}

int grid_for(int n_items) {
  int sms = 0;
  if (sm_count(&sms) != KQ_OK || sms <= 0) sms = 148;
  const int want = (n_items + kAuxThreads - 1) / kAuxThreads;
  const int cap = sms * 8;
  return want < cap ? (want > 0 ? want : 1) : cap;
}

}  // namespace
}  // namespace kq

extern "C" {

int kq_expand_params(const float* params, int64_t d, float* T, void* stream) {
  if (int st = kq::check_shape(1, d, 0, "kq_expand_params")) return st;
  if (!params || !T) return kq::fail(KQ_ERR_INVALID_ARG, "kq_expand_params: NULL pointer");
  if (!kq::aligned(params, 4) || !kq::aligned(T, 4))
    return kq::fail(KQ_ERR_ALIGNMENT, "kq_expand_params: pointers must be 4-byte aligned");
  const int64_t nb = d / 32;
  if (nb > (1 << 20)) return kq::fail(KQ_ERR_UNSUPPORTED, "kq_expand_params: d too large");
  const int total = (int)(nb * 1024);
  unsigned int* devstat = nullptr;
  if (int st = kq::device_status_address(&devstat)) return st;
  kq::expand_kernel<<<kq::grid_for(total), kq::kAuxThreads, 0, kq::as_stream(stream)>>>(
      params, (int)nb, T, devstat);
  return kq::check_launch("expand_kernel launch");
}

int kq_fold_weights(const float* W, int64_t N, int64_t d, const float* params, float* W_out,
                    void* stream) {
  if (int st = kq::check_shape(N, d, 0, "kq_fold_weights")) return st;
  if (N == 0) return KQ_OK;
  if (!W || !params || !W_out) return kq::fail(KQ_ERR_INVALID_ARG, "kq_fold_weights: NULL pointer");
  if (!kq::aligned(W, 16) || !kq::aligned(W_out, 16))
    return kq::fail(KQ_ERR_ALIGNMENT, "kq_fold_weights: W and W_out must be 16-byte aligned");
  if (!kq::aligned(params, 4))
    return kq::fail(KQ_ERR_ALIGNMENT, "kq_fold_weights: params must be 4-byte aligned");
  if (W != W_out) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(W), b = reinterpret_cast<uintptr_t>(W_out);
    const uintptr_t n = (uintptr_t)(N * d) * sizeof(float);
    if (a < b + n && b < a + n)
      return kq::fail(KQ_ERR_INVALID_ARG, "kq_fold_weights: W and W_out overlap partially");
  }
  const int nb = (int)(d / 32);
  const int n_blocks = (int)(N * nb);
  unsigned int* devstat = nullptr;
  if (int st = kq::device_status_address(&devstat)) return st;
  int sms = 0;
  if (int st = kq::sm_count(&sms)) return st;
  const int warps_per_cta = kq::kAuxThreads / 32;
  if (nb % 32 == 0) {
    // a whole number of warps per column group, enough to fill the device
    const int n_cg = nb / 32;
    int64_t groups_per_cg = (int64_t)sms * 8 * warps_per_cta / n_cg;
    if (groups_per_cg > N) groups_per_cg = N;
    if (groups_per_cg < 1) groups_per_cg = 1;
    int64_t warps = groups_per_cg * n_cg;
    const int64_t ctas = (warps + warps_per_cta - 1) / warps_per_cta;   // >= n_cg warps
    kq::fold_coalesced_kernel<true><<<(unsigned)ctas, kq::kAuxThreads, 0, kq::as_stream(stream)>>>(
        W, params, (int)N, nb, n_blocks, W_out, devstat);
  } else {
    const int pieces = (n_blocks + 31) / 32;
    int ctas = (pieces + warps_per_cta - 1) / warps_per_cta;
    if (ctas > sms * 8) ctas = sms * 8;
    kq::fold_coalesced_kernel<false><<<(unsigned)ctas, kq::kAuxThreads, 0, kq::as_stream(stream)>>>(
        W, params, (int)N, nb, n_blocks, W_out, devstat);
  }
  return kq::check_launch("fold_coalesced_kernel launch");
}

int kq_quantize_weights(const float* W, int64_t N, int64_t d, const float* params,
                        uint8_t* codes, uint8_t* scales, void* stream) {
  if (int st = kq::check_shape(N, d, 0, "kq_quantize_weights")) return st;
  if (N == 0) return KQ_OK;
  if (!W || !params || !codes || !scales)
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_quantize_weights: NULL pointer");
  if (!kq::aligned(W, 16) || !kq::aligned(codes, 16))
    return kq::fail(KQ_ERR_ALIGNMENT, "kq_quantize_weights: W and codes must be 16-byte aligned");
  if (!kq::aligned(params, 4))
    return kq::fail(KQ_ERR_ALIGNMENT, "kq_quantize_weights: params must be 4-byte aligned");
  const int nb = (int)(d / 32);
  const int n_blocks = (int)(N * nb);
  unsigned int* devstat = nullptr;
  if (int st = kq::device_status_address(&devstat)) return st;
  if (nb % 32 == 0) {
    // column-stationary: a whole number of warps per 32-block column group
    int sms = 0;
    if (int st = kq::sm_count(&sms)) return st;
    const int n_cg = nb / 32;
    const int64_t warps_want = (int64_t)sms * 8 * (kq::kAuxThreads / 32);
    int64_t rstep = warps_want / n_cg;
    if (rstep < 1) rstep = 1;
    if (rstep > N) rstep = N;
    const int64_t warps = rstep * n_cg;
    const int64_t blocks = (warps + kq::kAuxThreads / 32 - 1) / (kq::kAuxThreads / 32);
    kq::fold_quant_cs_kernel<<<(unsigned)blocks, kq::kAuxThreads, 0, kq::as_stream(stream)>>>(
        W, params, (int)N, nb, (int)rstep, codes, scales, devstat);
    return kq::check_launch("fold_quant_cs_kernel launch");
  }
  // one warp per 32 blocks
  const int64_t lanes = (int64_t)((n_blocks + 31) / 32) * 32;
  kq::fold_quant_kernel<<<kq::grid_for((int)lanes), kq::kAuxThreads, 0, kq::as_stream(stream)>>>(
      W, params, nb, n_blocks, codes, scales, devstat);
  return kq::check_launch("fold_quant_kernel launch");
}

int kq_row_sum(const void* x, int x_dtype, int64_t M, int64_t d, float scale, float* out, void* stream) {
  if (int st = kq::check_shape(M, d, 0, "kq_row_sum")) return st;
  if (x_dtype != KQ_DTYPE_BF16 && x_dtype != KQ_DTYPE_F32)
    return kq::fail(KQ_ERR_DTYPE, "kq_row_sum: x_dtype = %d", x_dtype);
  if (M == 0) return KQ_OK;
  if (!x || !out) return kq::fail(KQ_ERR_INVALID_ARG, "kq_row_sum: NULL pointer");
  if (!kq::aligned(x, 16) || !kq::aligned(out, 4))
    return kq::fail(KQ_ERR_ALIGNMENT, "kq_row_sum: x must be 16-byte and out 4-byte aligned");
  const int64_t lanes = M * 32;
  kq::row_sum_kernel<<<kq::grid_for(lanes > (1 << 30) ? (1 << 30) : (int)lanes), kq::kAuxThreads, 0,
                       kq::as_stream(stream)>>>(x, x_dtype == KQ_DTYPE_BF16, (int)M, (int)d, scale, out);
  return kq::check_launch("row_sum_kernel launch");
}

int kq_dequant(const uint8_t* codes, const uint8_t* scales, int64_t M, int64_t d, float* out,
               void* stream) {
  if (int st = kq::check_shape(M, d, 0, "kq_dequant")) return st;
  if (M == 0) return KQ_OK;
  if (!codes || !scales || !out) return kq::fail(KQ_ERR_INVALID_ARG, "kq_dequant: NULL pointer");
  if (!kq::aligned(codes, 16) || !kq::aligned(out, 16))
    return kq::fail(KQ_ERR_ALIGNMENT, "kq_dequant: codes and out must be 16-byte aligned");
  const int n_blocks = (int)(M * (d / 32));
  kq::dequant_kernel<<<kq::grid_for(n_blocks), kq::kAuxThreads, 0, kq::as_stream(stream)>>>(
      codes, scales, n_blocks, out);
  return kq::check_launch("dequant_kernel launch");
}

}  // extern "C"
