// Tensor-core KroQuant quantizer for bf16 activations (tcgen05 + TMEM).
//
// The per-block transform y = T_j x (a 32 x 32 contraction per token and
// block column) runs on the 5th-generation tensor cores as small GEMMs --
// the "small tensor-core GEMMs" option of the method -- and the SIMT warps
// only encode.  Exactness: x is bf16 (an exact operand); T_j is expanded in
// fp32 and split into three bf16 terms T = T_hi + T_mid + T_lo (residual
// below 2^-24 |T|), each multiplied exactly and accumulated in fp32 in
// tensor memory.
//
// Work split.  Block columns are cut into NC groups of C <= 4 (C = the
// largest divisor of nb not above 4).  A work unit is one group x one tile
// of 128 token rows; units are numbered group-major and every CTA (one per
// SM) takes one contiguous, balanced range of them, so that it meets at most
// three groups and keeps their T splits resident in shared memory.  A unit
// arrives by one 3-D TMA load of the view [nb][M][32] (box 32 x 128 x C):
// each block column lands as 128 contiguous 64-byte rows with the 64-byte
// swizzle, which is the canonical K-major SW64 operand layout of
// tcgen05.mma.
//
// Roles (320 threads):
//   warp 8, lane 0: TMA producer (S shared-memory stages, S * C * 8 KiB <= 128 KiB,
//                   plus an L2 prefetch of the unit S ahead);
//   warp 9        : allocates tensor memory; lane 0 issues the MMAs:
//                   per block column jj: 3 splits x 2 K-steps of
//                   M=128 x N=32 x K=16 into accumulator columns jj*32..;
//                   four accumulators of 128 columns;
//   warps 0..7    : epilogue.  Warp w reads TMEM lanes 32*(w%4).. (its token
//                   rows) for half (w/4) of the unit's block columns with
//                   tcgen05.ld 32x32b.x32 (one token's block per thread),
//                   hands the accumulator back and encodes.  The unit's codes
//                   are staged in shared memory (64-byte swizzle) and leave
//                   by one TMA tensor store; its scale bytes leave row by row.
//                   (The TMEM layout puts one token row in each thread, so
//                   direct stores would scatter every warp's writes over 32
//                   rows.)
// Every mbarrier wait is bounded; a wait that runs out sets the device status
// word and the CTA drains its copies and MMAs and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "kq.h"
#include "kq_device.cuh"
#include "kq_host.h"
#include "kq_tc.h"

namespace kq {
namespace tc {

constexpr int kEpiWarps = 8;
constexpr int kThreads = (kEpiWarps + 2) * 32;
constexpr int kProducerWarp = kEpiWarps;
constexpr int kMmaWarp = kEpiWarps + 1;
constexpr int kRows = 128;         // MMA M = token rows per unit
constexpr int kMaxC = 4;
constexpr int kMaxGroups = 3;      // table slots: column groups one CTA may meet
constexpr int kAcc = 4;            // accumulator buffers
constexpr int kAccCols = 128;      // TMEM columns per accumulator (C * 32 used)
constexpr int kTmemCols = kAcc * kAccCols;
constexpr int kStageBudget = 128 * 1024;
constexpr int kMaxStages = 16;

// UMMA instruction descriptor: D fp32, A and B bf16, both K-major, N = 32, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((32u >> 3) << 17) |
                            ((128u >> 4) << 24);

// Shared-memory matrix descriptor of a K-major, 64-byte-swizzled operand
// (8-row atoms of 64-byte rows, 512 bytes apart), sm_100 version field 1.
__device__ __forceinline__ uint64_t sw64_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(512 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)4 << 61);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(kIdesc), "r"(accum)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// 32 consecutive fp32 accumulator columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float2 (&v)[16]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
}

// Two blocks' accumulators with both loads in flight before one wait.
__device__ __forceinline__ void tmem_ld32x2(uint32_t t0, uint32_t t1, float2 (&v0)[16], float2 (&v1)[16]) {
  uint32_t r[32], s[32];
#define KQ_TLD(dst, addr)                                                                          \
  asm volatile(                                                                                    \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "                                                    \
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "                    \
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"   \
      : "=r"(dst[0]), "=r"(dst[1]), "=r"(dst[2]), "=r"(dst[3]), "=r"(dst[4]), "=r"(dst[5]),        \
        "=r"(dst[6]), "=r"(dst[7]), "=r"(dst[8]), "=r"(dst[9]), "=r"(dst[10]), "=r"(dst[11]),      \
        "=r"(dst[12]), "=r"(dst[13]), "=r"(dst[14]), "=r"(dst[15]), "=r"(dst[16]), "=r"(dst[17]),  \
        "=r"(dst[18]), "=r"(dst[19]), "=r"(dst[20]), "=r"(dst[21]), "=r"(dst[22]), "=r"(dst[23]),  \
        "=r"(dst[24]), "=r"(dst[25]), "=r"(dst[26]), "=r"(dst[27]), "=r"(dst[28]), "=r"(dst[29]),  \
        "=r"(dst[30]), "=r"(dst[31])                                                               \
      : "r"(addr))
  KQ_TLD(r, t0);
  KQ_TLD(s, t1);
#undef KQ_TLD
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    v0[i] = make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
    v1[i] = make_float2(__uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1]));
  }
}


// Shared-memory layout (offsets from the 1024-aligned base).
struct Layout {
  int stages;        // S
  int stage_bytes;   // C * 128 * 64
  int table_off;     // kMaxGroups * C * 3 * 2048 bytes of T splits
  int fac_off;       // kMaxGroups * C * 5 float4 LU factors (set-up only)
  int out_off;       // two code tiles of 128 rows x C * 16 bytes (TMA store sources)
  int out_bytes;
  int sc_off;        // two scale tiles of 128 rows x C bytes
  int bar_off;       // 2 S + 2 kAcc barriers, abort flag, TMEM address
  int total;
};

__host__ __device__ inline Layout layout_for(int C) {
  Layout L;
  L.stage_bytes = C * kRows * 64;
  L.stages = kStageBudget / L.stage_bytes;
  if (L.stages > kMaxStages) L.stages = kMaxStages;
  L.table_off = L.stages * L.stage_bytes;
  L.fac_off = L.table_off + kMaxGroups * C * 3 * 2048;
  L.out_off = L.fac_off + 1024;
  L.out_bytes = ((kRows * C * 16) + 1023) & ~1023;
  L.sc_off = L.out_off + 2 * L.out_bytes;
  L.bar_off = L.sc_off + 2 * kRows * kMaxC;
  L.total = L.bar_off + 512;
  return L;
}

// Staging position of (token row r, block jj) in a code tile of C*16-byte rows.
// With C == 4 the rows are 64 bytes and the 64-byte swizzle (16-byte chunk ^=
// (r >> 1) & 3) keeps a warp's 32 row writes free of bank conflicts; the TMA
// store map uses the same swizzle.
__device__ __forceinline__ int out_offset(int C, int r, int jj) {
  return C == 4 ? r * 64 + ((jj ^ ((r >> 1) & 3)) << 4) : (r * C + jj) * 16;
}

__device__ __forceinline__ void tma_store_2d(const void* tmap, int c0, int c1, uint32_t src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
               ::"l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Barrier 1 among the epilogue warps only (the producer and MMA warps never
// take part).  epi_any also ORs a flag across them, so every epilogue warp
// takes the same branch after it and no warp is left waiting.
__device__ __forceinline__ void epi_barrier() {
  asm volatile("bar.sync 1, %0;" ::"r"(kEpiWarps * 32) : "memory");
}
__device__ __forceinline__ bool epi_any(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(kEpiWarps * 32)
      : "memory");
  return r != 0;
}

__global__ void __launch_bounds__(kThreads, 1)
tc_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap omap,
          const float* __restrict__ params,
          const TcGeometry geo, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
          unsigned int* devstat) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int C = geo.C;
  const Layout L = layout_for(C);
  const int S = L.stages;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  const uint32_t full0 = smem_addr(&bars[0]), empty0 = smem_addr(&bars[S]);
  const uint32_t accf0 = smem_addr(&bars[2 * S]), acce0 = smem_addr(&bars[2 * S + kAcc]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.bar_off + 384);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.bar_off + 448);
  const uint32_t table = smem_addr(smem + L.table_off);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_rt = geo.n_row_tiles;
  const int64_t U = (int64_t)geo.NC * n_rt;
  const int64_t u_begin = (int64_t)blockIdx.x * U / gridDim.x;
  const int64_t u_end = (int64_t)(blockIdx.x + 1) * U / gridDim.x;
  const int n_items = (int)(u_end - u_begin);
  const int g_first = (int)(u_begin / n_rt);
  const int n_groups = n_items > 0 ? (int)((u_end - 1) / n_rt) - g_first + 1 : 0;

  pdl_launch_dependents();
  if (tid == 0) {
    tma_prefetch_desc(&tmap);
    tma_prefetch_desc(&omap);
    for (int i = 0; i < S; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, 1);
    }
    for (int i = 0; i < kAcc; ++i) {
      mbar_init(accf0 + 8 * i, 1);
      mbar_init(acce0 + 8 * i, kEpiWarps);
    }
    *abort_flag = 0;
    mbar_init_fence();
    // L2 prefetch of the first units before the wait on the previous kernel
    // (a hint that changes no memory; the loads after the wait see that
    // kernel's writes, which land in L2)
    for (int it = 0; it < n_items && it < S; ++it) {
      const int64_t u = u_begin + it;
      const int g = (int)(u / n_rt), rt = (int)(u - (int64_t)g * n_rt);
      tma_prefetch_l2_3d(&tmap, 0, rt * kRows, g * C);
    }
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_wait_predecessor();
  __syncthreads();

  // The first S loads go out before the tables are built.
  const uint32_t tx = (uint32_t)L.stage_bytes;
  auto issue = [&](int it) {
    const int64_t u = u_begin + it;
    const int g = (int)(u / n_rt), rt = (int)(u - (int64_t)g * n_rt);
    const int s = it % S;
    mbar_arrive_expect_tx(full0 + 8 * s, tx);
    tma_load_3d(smem_addr(smem + s * L.stage_bytes), &tmap, 0, rt * kRows, g * C, full0 + 8 * s);
  };
  // L2 prefetch of a later unit: its bytes are on the way while the unit
  // waits for a free stage, so more than the stages' worth is in flight
  auto prefetch = [&](int it) {
    const int64_t u = u_begin + it;
    const int g = (int)(u / n_rt), rt = (int)(u - (int64_t)g * n_rt);
    tma_prefetch_l2_3d(&tmap, 0, rt * kRows, g * C);
  };
  if (warp == kProducerWarp && lane == 0) {
    for (int it = 0; it < n_items && it < S; ++it) issue(it);
    for (int it = S; it < n_items && it < 2 * S; ++it) prefetch(it);
  }

  // T splits of the groups this CTA meets: [slot][jj][part][n = output row][k],
  // bf16, 64-byte rows with the 64-byte swizzle (16-byte chunk ^= (n >> 1) & 3).
  // First the five LU factors of every block column, then one thread per
  // output row n expands T[n][.] = prod_m A_m[bit(n)][bit(.)] by Kronecker
  // doubling (factor 0 on the most significant index bit) and splits it.
  float4* fac = reinterpret_cast<float4*>(smem + L.fac_off);
  for (int i = tid; i < n_groups * C * 5; i += kThreads) {
    const int cj = i / 5, m = i - 5 * cj;   // cj = slot * C + jj
    const float* p = params + 15 * ((int64_t)g_first * C + cj) + 3 * m;
    if (lu_params_bad(p[0], p[1], p[2])) atomicOr(devstat, (unsigned)KQ_DEVSTAT_BAD_PARAMS);
    fac[i] = lu_factor(p[0], p[1], p[2]);
  }
  __syncthreads();
  for (int ri = tid; ri < n_groups * C * 32; ri += kThreads) {
    const int cj = ri >> 5, n = ri & 31;
    float t[32];
    t[0] = 1.0f;
#pragma unroll
    for (int m = 0; m < 5; ++m) {
      const float4 A = fac[cj * 5 + m];
      const bool hi_row = (n >> (4 - m)) & 1;
      const float a0 = hi_row ? A.z : A.x, a1 = hi_row ? A.w : A.y;
#pragma unroll
      for (int q = (1 << m) - 1; q >= 0; --q) {
        t[2 * q + 1] = __fmul_rn(t[q], a1);
        t[2 * q] = __fmul_rn(t[q], a0);
      }
    }
    uint8_t* rowp = smem + L.table_off + cj * 3 * 2048 + n * 64;
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      uint32_t w[3][4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = t[8 * ch + 2 * e], x1 = t[8 * ch + 2 * e + 1];
        const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
        const float r0 = x0 - __low2float(h), r1 = x1 - __high2float(h);
        const __nv_bfloat162 mid = __floats2bfloat162_rn(r0, r1);
        const __nv_bfloat162 lo = __floats2bfloat162_rn(r0 - __low2float(mid), r1 - __high2float(mid));
        w[0][e] = *reinterpret_cast<const uint32_t*>(&h);
        w[1][e] = *reinterpret_cast<const uint32_t*>(&mid);
        w[2][e] = *reinterpret_cast<const uint32_t*>(&lo);
      }
      const int off = ((ch ^ ((n >> 1) & 3))) << 4;
#pragma unroll
      for (int part = 0; part < 3; ++part)
        *reinterpret_cast<uint4*>(rowp + part * 2048 + off) =
            make_uint4(w[part][0], w[part][1], w[part][2], w[part][3]);
    }
  }
  // make the generic-proxy table writes visible to the tensor cores
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      int issued = n_items < S ? n_items : S;
      for (int it = S; it < n_items; ++it) {
        const int s = it % S;
        if (!mbar_wait_bounded(empty0 + 8 * s, (uint32_t)(it / S - 1) & 1u)) {
          *abort_flag = 1;
          atomicOr(devstat, (unsigned)KQ_DEVSTAT_WAIT_TIMEOUT);
          break;
        }
        if (*abort_flag) break;
        issue(it);
        issued = it + 1;
        if (it + S < n_items) prefetch(it + S);
      }
      // after an abort, let the copies still in flight land before the
      // shared memory goes away (on the normal path these return at once)
      if (*abort_flag) {
        const int lo = issued > S ? issued - S : 0;
        for (int it = lo; it < issued; ++it)
          (void)mbar_wait_bounded(full0 + 8 * (it % S), (uint32_t)(it / S) & 1u);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      int done = 0;
      for (int it = 0; it < n_items; ++it) {
        const int s = it % S, a = it % kAcc;
        const bool ok_full = mbar_wait_bounded(full0 + 8 * s, (uint32_t)(it / S) & 1u);
        const bool ok_acc =
            it < kAcc || mbar_wait_bounded(acce0 + 8 * a, (uint32_t)(it / kAcc - 1) & 1u);
        if (!ok_full || !ok_acc || *abort_flag) {
          *abort_flag = 1;
          atomicOr(devstat, (unsigned)KQ_DEVSTAT_WAIT_TIMEOUT);
          break;
        }
        fence_after_sync();
        const int64_t u = u_begin + it;
        const int slot = (int)(u / n_rt) - g_first;
        const uint32_t a_base = smem_addr(smem + s * L.stage_bytes);
        const uint32_t t_base = table + (uint32_t)(slot * C * 3 * 2048);
        for (int jj = 0; jj < C; ++jj) {
          const uint32_t d = tmem_base + (uint32_t)(a * kAccCols + jj * 32);
#pragma unroll
          for (int part = 0; part < 3; ++part) {
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
              const uint64_t adesc = sw64_desc(a_base + jj * (kRows * 64) + ks * 32);
              const uint64_t bdesc = sw64_desc(t_base + (jj * 3 + part) * 2048 + ks * 32);
              mma_bf16(d, adesc, bdesc, (part | ks) != 0);
            }
          }
        }
        mma_commit(empty0 + 8 * s);   // shared-memory stage free once these MMAs are done
        mma_commit(accf0 + 8 * a);    // accumulator ready for the epilogue
        done = it + 1;
      }
      // after an abort, wait (bounded) for the last MMAs before TMEM and the
      // stages are released; MMAs complete in issue order
      if (*abort_flag && done > 0)
        (void)mbar_wait_bounded(accf0 + 8 * ((done - 1) % kAcc), (uint32_t)((done - 1) / kAcc) & 1u);
    }
  } else {
    // epilogue warps: the codes of a unit are staged in shared memory and
    // written by one TMA tensor store (128 rows x C * 16 bytes), the scale
    // bytes row by row; two staging buffers alternate
    const int q = warp & 3;                 // TMEM lane quarter = token rows 32q..32q+31
    const int h = warp >> 2;                // which half of the unit's block columns
    const int jj_lo = (h * C) / 2, jj_hi = ((h + 1) * C) / 2;
    const int cnt = jj_hi - jj_lo;
    const int nb = geo.nb;
    const int r_local = 32 * q + lane;      // token row inside the unit
    for (int it = 0; it < n_items; ++it) {
      const int a = it % kAcc, buf = it & 1;
      const bool ok = mbar_wait_bounded(accf0 + 8 * a, (uint32_t)(it / kAcc) & 1u);
      if (!ok) atomicOr(devstat, (unsigned)KQ_DEVSTAT_WAIT_TIMEOUT);
      // the TMA store that last read this staging buffer (item it - 2) is done
      if (tid == 0) bulk_wait_read_1();
      // one decision for all epilogue warps (also the staging-buffer barrier)
      if (epi_any(!ok || *abort_flag)) {
        *abort_flag = 1;
        break;
      }
      fence_after_sync();
      const int64_t u = u_begin + it;
      const int g = (int)(u / n_rt), rt = (int)(u - (int64_t)g * n_rt);
      const uint32_t tq = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * kAccCols);
      float2 v0[16], v1[16];
      if (cnt == 2) {
        tmem_ld32x2(tq + (uint32_t)(jj_lo * 32), tq + (uint32_t)((jj_lo + 1) * 32), v0, v1);
      } else if (cnt == 1) {
        tmem_ld32(tq + (uint32_t)(jj_lo * 32), v0);
      }
      // this warp's reads of accumulator a are complete: hand it back
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce0 + 8 * a);
      uint8_t* stage_out = smem + L.out_off + buf * L.out_bytes;
      uint8_t* stage_sc = smem + L.sc_off + buf * (kRows * kMaxC);
      if (cnt > 0) {
        uint4 p0;
        stage_sc[r_local * C + jj_lo] = (uint8_t)mxfp4_encode32(v0, p0);
        *reinterpret_cast<uint4*>(stage_out + out_offset(C, r_local, jj_lo)) = p0;
        if (cnt == 2) {
          uint4 p1;
          stage_sc[r_local * C + jj_lo + 1] = (uint8_t)mxfp4_encode32(v1, p1);
          *reinterpret_cast<uint4*>(stage_out + out_offset(C, r_local, jj_lo + 1)) = p1;
        }
      }
      // generic-proxy writes -> visible to the TMA store, then all warps done
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      epi_barrier();
      if (tid == 0) {
        tma_store_2d(&omap, g * C * 16, rt * kRows, smem_addr(stage_out));
        bulk_commit();
      }
      // scale bytes: one thread per token row writes the unit's C bytes
      if (tid < kRows) {
        const int row = rt * kRows + tid;
        if (row < geo.M) {
          uint8_t* dst = scales + (size_t)row * nb + (size_t)g * C;
          const uint8_t* srcp = stage_sc + tid * C;
          if (C == 4 && (reinterpret_cast<uintptr_t>(dst) & 3) == 0) {
            *reinterpret_cast<uint32_t*>(dst) = *reinterpret_cast<const uint32_t*>(srcp);
          } else {
            for (int c = 0; c < C; ++c) dst[c] = srcp[c];
          }
        }
      }
    }
    if (tid == 0) bulk_wait_all();
  }

  fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    fence_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemCols)
                 : "memory");
  }
}

}  // namespace tc

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace {

int tc_choose_C(int nb) {
  for (int c = nb < tc::kMaxC ? nb : tc::kMaxC; c > 1; --c)
    if (nb % c == 0) return c;
  return 1;
}

// Most column groups any CTA meets when U units are split into G balanced
// contiguous ranges.
int max_groups_met(int64_t U, int64_t G, int n_rt) {
  int worst = 0;
  for (int64_t i = 0; i < G; ++i) {
    const int64_t b = i * U / G, e = (i + 1) * U / G;
    if (e > b) {
      const int span = (int)((e - 1) / n_rt - b / n_rt + 1);
      if (span > worst) worst = span;
    }
  }
  return worst;
}

PFN_cuTensorMapEncodeTiled_v12000 tc_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

constexpr int kMaxDevices = 64;

}  // namespace

int tc_quantize(const void* x, int64_t M, int64_t d, const float* params, uint8_t* codes,
                uint8_t* scales, cudaStream_t stream) {
  TcGeometry geo;
  geo.nb = (int)(d / 32);
  geo.C = tc_choose_C(geo.nb);
  geo.NC = geo.nb / geo.C;
  geo.M = (int)M;
  geo.n_row_tiles = (int)((M + tc::kRows - 1) / tc::kRows);
  const tc::Layout L = tc::layout_for(geo.C);
  const size_t smem = 1024 + (size_t)L.total;
  auto kern = tc::tc_kernel;

  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return cuda_fail(err, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(KQ_ERR_UNSUPPORTED, "device ordinal %d", dev);
  static std::once_flag attr_once[kMaxDevices];
  static cudaError_t attr_err[kMaxDevices];
  std::call_once(attr_once[dev], [&] {
    int optin = 0;
    attr_err[dev] = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (attr_err[dev] == cudaSuccess)
      attr_err[dev] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  });
  if (attr_err[dev] != cudaSuccess) return cuda_fail(attr_err[dev], "cudaFuncSetAttribute");

  PFN_cuTensorMapEncodeTiled_v12000 enc = tc_encoder();
  if (!enc) return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled not found in the CUDA driver");
  CUtensorMap tm;
  // view [nb][M][32]: dim0 = 32 elements, dim1 = rows (stride d*2), dim2 = blocks (stride 64)
  const cuuint64_t dims[3] = {32, (cuuint64_t)M, (cuuint64_t)geo.nb};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, 64};
  const cuuint32_t box[3] = {32, (cuuint32_t)tc::kRows, (cuuint32_t)geo.C};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), dims, strides,
                         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);

  CUtensorMap om;
  {
    // codes [M][d/2] bytes; box = C*16 bytes x 128 rows
    const cuuint64_t odims[2] = {(cuuint64_t)d / 2, (cuuint64_t)M};
    const cuuint64_t ostrides[1] = {(cuuint64_t)d / 2};
    const cuuint32_t obox[2] = {(cuuint32_t)(geo.C * 16), (cuuint32_t)tc::kRows};
    const cuuint32_t oestr[2] = {1, 1};
    const CUresult r2 = enc(&om, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, codes, odims, ostrides, obox, oestr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE,
                            geo.C == 4 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r2 != CUDA_SUCCESS)
      return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled (codes) failed (CUresult %d)", (int)r2);
  }

  int sms = 0;
  if (int st = sm_count(&sms)) return st;
  const int64_t U = (int64_t)geo.NC * geo.n_row_tiles;
  int64_t grid = U < sms ? U : sms;
  // every CTA keeps the T splits of the groups it meets: at most kMaxGroups
  while (max_groups_met(U, grid, geo.n_row_tiles) > tc::kMaxGroups) grid += sms;
  if (grid > U) grid = U;
  if (grid > 0x7fffffff) return fail(KQ_ERR_UNSUPPORTED, "kq_quantize_tc: grid too large");

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(tc::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  unsigned int* devstat = nullptr;
  if (int st = device_status_address(&devstat)) return st;
  err = cudaLaunchKernelEx(&cfg, kern, tm, om, params, geo, codes, scales, devstat);
  if (err != cudaSuccess) return cuda_fail(err, "tc_kernel launch");
  return check_launch("tc_kernel launch");
}

}  // namespace kq

extern "C" int kq_quantize_tc(const void* x, int x_dtype, int64_t M, int64_t d,
                              const float* params, uint8_t* codes, uint8_t* scales,
                              void* stream) {
  const char* fn = "kq_quantize_tc";
  if (int st = kq::check_shape(M, d, KQ_MAX_D, fn)) return st;
  if (x_dtype != KQ_DTYPE_BF16)
    return kq::fail(KQ_ERR_DTYPE, "%s: only bf16 input (x_dtype = %d)", fn, x_dtype);
  if (M == 0) return KQ_OK;
  if (!x || !params || !codes || !scales) return kq::fail(KQ_ERR_INVALID_ARG, "%s: NULL pointer", fn);
  if (!kq::aligned(x, 16)) return kq::fail(KQ_ERR_ALIGNMENT, "%s: x must be 16-byte aligned", fn);
  if (!kq::aligned(params, 4)) return kq::fail(KQ_ERR_ALIGNMENT, "%s: parameters must be 4-byte aligned", fn);
  if (!kq::aligned(codes, 16)) return kq::fail(KQ_ERR_ALIGNMENT, "%s: codes must be 16-byte aligned", fn);
  return kq::tc_quantize(x, M, d, params, codes, scales, kq::as_stream(stream));
}
