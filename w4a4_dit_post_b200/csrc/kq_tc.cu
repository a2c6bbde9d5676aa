// Tensor-core KroQuant quantizer for bf16 activations (tcgen05 + TMEM).
//
// The per-block transform y = T_j x (a 32 x 32 contraction per token and
// block column) runs on the 5th-generation tensor cores as small GEMMs --
// the "small tensor-core GEMMs" of the method -- and the SIMT warps only
// encode.  Exactness: x is bf16 (exact operand); T_j is expanded in fp32 and
// split into three bf16 terms T = T_hi + T_mid + T_lo (residual below 2^-27
// |T|), each multiplied exactly and accumulated in fp32 in tensor memory.
//
// Work split.  Block columns are cut into NC groups of C <= 8 (C = the
// largest divisor of nb not above 8); a CTA owns one group for its life
// (grid = a multiple of NC, one CTA per SM) and walks row tiles of 128 rows.
// A tile arrives by one 3-D TMA load of the view [nb][M][32] (box 32 x 128 x
// C): each block column lands as 128 contiguous 64-byte rows with the 64-byte
// swizzle, which is the canonical K-major SW64 operand layout of tcgen05.mma.
// The CTA's T splits (C x 3 x 2 KiB, same layout) are built once in shared
// memory from the LU parameters.
//
// Roles (576 threads):
//   warp 16, lane 0: TMA producer (two shared-memory stages);
//   warp 17        : allocates tensor memory; lane 0 issues the MMAs:
//                    per block column jj: 3 splits x 2 K-steps of
//                    M=128 x N=32 x K=16 into accumulator columns jj*32..;
//                    two accumulators of C*32 columns (double buffer);
//   warps 0..15    : epilogue.  Warp w reads TMEM lanes 32*(w%4).. (its token
//                    rows) for the block columns of quarter (w/4) of the group
//                    with tcgen05.ld 32x32b.x32 (one token's block per
//                    thread, up to two loads in flight), encodes into a
//                    swizzled shared tile, and one thread stores the tile
//                    of codes with a TMA tensor store.
// Every mbarrier wait is bounded; a wait that runs out sets the device status
// word and the CTA drains and exits.
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

constexpr int kEpiWarps = 16;
constexpr int kThreads = (kEpiWarps + 2) * 32;
constexpr int kProducerWarp = kEpiWarps;
constexpr int kMmaWarp = kEpiWarps + 1;
constexpr int kRows = 128;        // MMA M = token rows per tile
constexpr int kMaxC = 8;
constexpr int kStages = 2;
constexpr int kTmemCols = 512;    // two accumulators of up to 8 x 32 columns

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
  int stage_bytes;   // C * 128 * 64
  int table_off;     // after the stages; C * 3 * 2048 bytes
  int out_off;       // two code staging buffers of 128 x C*16 bytes (1024-aligned)
  int out_bytes;
  int sc_off;        // scale staging, 128 x C bytes
  int bar_off;       // barriers and flags
  int total;
};

__host__ __device__ inline Layout layout_for(int C) {
  Layout L;
  L.stage_bytes = C * kRows * 64;
  L.table_off = kStages * L.stage_bytes;
  L.out_off = L.table_off + C * 3 * 2048;
  L.out_bytes = ((kRows * C * 16) + 1023) & ~1023;
  L.sc_off = L.out_off + 2 * L.out_bytes;       // scale bytes of one tile: 128 x C
  L.bar_off = L.sc_off + ((kRows * C + 127) & ~127);
  L.total = L.bar_off + 256;
  return L;
}

// Staging position of (token row r, block jj) in a code tile of C*16-byte rows.
// With C == 8 the rows are 128 bytes and the 128-byte swizzle (chunk ^ r % 8)
// keeps the per-row 16-byte writes conflict-free; the TMA store map matches.
__device__ __forceinline__ int out_offset(int C, int r, int jj) {
  return C == 8 ? r * 128 + ((jj ^ (r & 7)) << 4) : (r * C + jj) * 16;
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
// takes the same branch after it (no warp can leave another waiting).
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

template <bool kTransformOnly>
__global__ void __launch_bounds__(kThreads, 1)
tc_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap omap,
          const float* __restrict__ params,
          const TcGeometry geo, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
          float* __restrict__ y_out, unsigned int* devstat) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int C = geo.C;
  const Layout L = layout_for(C);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  // bars: full[2], empty[2], acc_full[2], acc_empty[2]
  const uint32_t full0 = smem_addr(&bars[0]), empty0 = smem_addr(&bars[2]);
  const uint32_t accf0 = smem_addr(&bars[4]), acce0 = smem_addr(&bars[6]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.bar_off + 64);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.bar_off + 128);
  const uint32_t table = smem_addr(smem + L.table_off);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int col_group = blockIdx.x % geo.NC;
  const int row_step = gridDim.x / geo.NC;
  const int rt_first = blockIdx.x / geo.NC;
  const int j0 = col_group * C;
  const int n_items = rt_first < geo.n_row_tiles
                          ? (geo.n_row_tiles - rt_first + row_step - 1) / row_step
                          : 0;

  pdl_launch_dependents();
  if (tid == 0) {
    tma_prefetch_desc(&tmap);
    if (!kTransformOnly) tma_prefetch_desc(&omap);
    for (int i = 0; i < 2; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, 1);
      mbar_init(accf0 + 8 * i, 1);
      mbar_init(acce0 + 8 * i, kEpiWarps);
    }
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_wait_predecessor();

  // T splits of the C block columns: [jj][part][n = output row][k], bf16,
  // 64-byte rows with the 64-byte swizzle (chunk ^= (n >> 1) & 3).  The five
  // factors of each column are computed once (C * 5 threads), then each
  // thread forms entries T[n][k] = prod_m A_m[bit][bit] and splits them.
  float4* fac = reinterpret_cast<float4*>(smem + L.out_off);   // staging area, free until the epilogue
  for (int i = tid; i < C * 5; i += kThreads) {
    const int jj = i / 5, m = i - 5 * jj;
    const float* p = params + 15 * (j0 + jj) + 3 * m;
    fac[i] = lu_factor(p[0], p[1], p[2]);
  }
  __syncthreads();
  for (int i = tid; i < C * 1024; i += kThreads) {
    const int jj = i >> 10, n = (i >> 5) & 31, k = i & 31;
    float t = 1.0f;
#pragma unroll
    for (int m = 0; m < 5; ++m) {
      const float4 A = fac[jj * 5 + m];
      const int bn = (n >> (4 - m)) & 1, bk = (k >> (4 - m)) & 1;
      t = __fmul_rn(t, bn ? (bk ? A.w : A.z) : (bk ? A.y : A.x));
    }
    const __nv_bfloat16 hi = __float2bfloat16_rn(t);
    const float r1 = t - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
    const int off = n * 64 + ((((k >> 3) ^ ((n >> 1) & 3))) << 4) + (k & 7) * 2;
    __nv_bfloat16* base = reinterpret_cast<__nv_bfloat16*>(smem + L.table_off + jj * 3 * 2048);
    base[(0 * 2048 + off) / 2] = hi;
    base[(1 * 2048 + off) / 2] = mid;
    base[(2 * 2048 + off) / 2] = lo;
  }
  // make the generic-proxy table writes visible to the tensor cores
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t acc_cols = (uint32_t)(C * 32);

  if (warp == kProducerWarp) {
    if (lane == 0) {
      const uint32_t tx = (uint32_t)L.stage_bytes;
      for (int it = 0; it < n_items; ++it) {
        const int s = it & 1;
        if (it >= 2 && !mbar_wait_bounded(empty0 + 8 * s, (uint32_t)((it >> 1) - 1) & 1u)) {
          *abort_flag = 1;
          atomicOr(devstat, (unsigned)KQ_DEVSTAT_WAIT_TIMEOUT);
          break;
        }
        if (*abort_flag) break;
        const int rt = rt_first + it * row_step;
        mbar_arrive_expect_tx(full0 + 8 * s, tx);
        tma_load_3d(smem_addr(smem + s * L.stage_bytes), &tmap, 0, rt * kRows, j0, full0 + 8 * s);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      for (int it = 0; it < n_items; ++it) {
        const int s = it & 1, a = it & 1;
        const bool ok_full = mbar_wait_bounded(full0 + 8 * s, (uint32_t)(it >> 1) & 1u);
        const bool ok_acc = it < 2 || mbar_wait_bounded(acce0 + 8 * a, (uint32_t)((it >> 1) - 1) & 1u);
        if (!ok_full || !ok_acc || *abort_flag) {
          *abort_flag = 1;
          atomicOr(devstat, (unsigned)KQ_DEVSTAT_WAIT_TIMEOUT);
          break;
        }
        fence_after_sync();
        const uint32_t a_base = smem_addr(smem + s * L.stage_bytes);
        for (int jj = 0; jj < C; ++jj) {
          const uint32_t d = tmem_base + (uint32_t)a * acc_cols + (uint32_t)(jj * 32);
#pragma unroll
          for (int part = 0; part < 3; ++part) {
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
              const uint64_t adesc = sw64_desc(a_base + jj * (kRows * 64) + ks * 32);
              const uint64_t bdesc = sw64_desc(table + (jj * 3 + part) * 2048 + ks * 32);
              mma_bf16(d, adesc, bdesc, (part | ks) != 0);
            }
          }
        }
        mma_commit(empty0 + 8 * s);   // shared-memory stage free once these MMAs are done
        mma_commit(accf0 + 8 * a);    // accumulator ready for the epilogue
      }
    }
  } else {
    // epilogue warps
    const int q = warp & 3;                 // TMEM lane quarter = token rows 32q..32q+31
    const int slot = warp >> 2;             // which quarter of the group's block columns
    const int jj_lo = (slot * C) / 4;
    const int jj_hi = ((slot + 1) * C) / 4;
    const int nb = geo.nb;
    const int r_local = 32 * q + lane;      // token row inside the tile
    for (int it = 0; it < n_items; ++it) {
      const int a = it & 1;
      const bool ok = mbar_wait_bounded(accf0 + 8 * a, (uint32_t)(it >> 1) & 1u);
      if (!ok) atomicOr(devstat, (unsigned)KQ_DEVSTAT_WAIT_TIMEOUT);
      // the TMA store that last read this staging buffer (item it - 2) is done
      if (!kTransformOnly && tid == 0) bulk_wait_read_1();
      // one decision for all epilogue warps (also the staging-buffer barrier)
      if (epi_any(!ok || *abort_flag)) {
        *abort_flag = 1;
        break;
      }
      fence_after_sync();
      const int rt = rt_first + it * row_step;
      const int row = rt * kRows + r_local;
      uint8_t* stage_out = smem + L.out_off + a * L.out_bytes;
      uint8_t* stage_sc = smem + L.sc_off;
      const uint32_t tq = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)a * acc_cols;
      auto emit = [&](int jj, const float2 (&v)[16]) {
        if constexpr (kTransformOnly) {
          if (row < geo.M) {
            float4* dst = reinterpret_cast<float4*>(y_out + ((size_t)row * nb + j0 + jj) * 32);
#pragma unroll
            for (int t = 0; t < 8; ++t)
              dst[t] = make_float4(v[2 * t].x, v[2 * t].y, v[2 * t + 1].x, v[2 * t + 1].y);
          }
        } else {
          uint4 packed;
          const uint32_t byte = mxfp4_encode32(v, packed);
          *reinterpret_cast<uint4*>(stage_out + out_offset(C, r_local, jj)) = packed;
          stage_sc[r_local * C + jj] = (uint8_t)byte;
        }
      };
      int jj = jj_lo;
      for (; jj + 1 < jj_hi; jj += 2) {
        float2 v0[16], v1[16];
        tmem_ld32x2(tq + (uint32_t)(jj * 32), tq + (uint32_t)((jj + 1) * 32), v0, v1);
        emit(jj, v0);
        emit(jj + 1, v1);
      }
      if (jj < jj_hi) {
        float2 v[16];
        tmem_ld32(tq + (uint32_t)(jj * 32), v);
        emit(jj, v);
      }
      // this warp's reads of accumulator a are complete: hand it back
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce0 + 8 * a);
      if (!kTransformOnly) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        epi_barrier();
        if (tid == 0) {
          tma_store_2d(&omap, j0 * 16, rt * kRows, smem_addr(stage_out));
          bulk_commit();
        }
        // scale bytes: consecutive threads write consecutive bytes of a row
        for (int i = tid; i < kRows * C; i += kEpiWarps * 32) {
          const int r = i / C, c = i - r * C;
          const int grow = rt * kRows + r;
          if (grow < geo.M) scales[(size_t)grow * nb + j0 + c] = stage_sc[i];
        }
      }
    }
    if (!kTransformOnly && tid == 0) bulk_wait_all();
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

template <bool kTransformOnly>
int tc_launch(const void* x, int64_t M, int64_t d, const float* params, uint8_t* codes,
              uint8_t* scales, float* y, cudaStream_t stream) {
  TcGeometry geo;
  geo.nb = (int)(d / 32);
  geo.C = tc_choose_C(geo.nb);
  geo.NC = geo.nb / geo.C;
  geo.M = (int)M;
  geo.n_row_tiles = (int)((M + tc::kRows - 1) / tc::kRows);
  const tc::Layout L = tc::layout_for(geo.C);
  const size_t smem = 1024 + (size_t)L.total;
  auto kern = tc::tc_kernel<kTransformOnly>;

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
  memset(&om, 0, sizeof(om));
  if (!kTransformOnly) {
    // codes [M][d/2] bytes; box = C*16 bytes x 128 rows
    const cuuint64_t odims[2] = {(cuuint64_t)d / 2, (cuuint64_t)M};
    const cuuint64_t ostrides[1] = {(cuuint64_t)d / 2};
    const cuuint32_t obox[2] = {(cuuint32_t)(geo.C * 16), (cuuint32_t)tc::kRows};
    const cuuint32_t oestr[2] = {1, 1};
    const CUresult r2 = enc(&om, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, codes, odims, ostrides, obox, oestr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE,
                            geo.C == 8 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r2 != CUDA_SUCCESS)
      return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled (codes) failed (CUresult %d)", (int)r2);
  }

  int sms = 0;
  if (int st = sm_count(&sms)) return st;
  int64_t per_group = sms / geo.NC;
  if (per_group < 1) per_group = 1;
  if (per_group > geo.n_row_tiles) per_group = geo.n_row_tiles;
  const int64_t grid = per_group * geo.NC;

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
  err = cudaLaunchKernelEx(&cfg, kern, tm, om, params, geo, codes, scales, y, devstat);
  if (err != cudaSuccess) return cuda_fail(err, "tc_kernel launch");
  return check_launch("tc_kernel launch");
}

}  // namespace

int tc_quantize(const void* x, int64_t M, int64_t d, const float* params, uint8_t* codes,
                uint8_t* scales, cudaStream_t stream) {
  return tc_launch<false>(x, M, d, params, codes, scales, nullptr, stream);
}

int tc_transform(const void* x, int64_t M, int64_t d, const float* params, float* y,
                 cudaStream_t stream) {
  return tc_launch<true>(x, M, d, params, nullptr, nullptr, y, stream);
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
