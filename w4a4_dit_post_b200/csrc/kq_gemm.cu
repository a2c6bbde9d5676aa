// The W4A4 linear layer on the quantised operands: Y = A B^T, where A [M, K]
// are MXFP4 activation codes (kq_quantize) and B [N, K] MXFP4 weight codes
// (kq_quantize_weights), each with one E8M0 scale per 32 values along K.
//
// The products run on the 5th-generation tensor cores with the block-scaled
// FP4 MMA (tcgen05.mma kind::mxf4, one scale per 32 elements): the E2M1 codes
// go in as stored (two per byte), the scales ride along in tensor memory, and
// the fp32 accumulator lives in tensor memory.
//
// Scale factors.  The MMA reads the scale of row m from tensor-memory lane m,
// column m / 32 of a 4-column group, byte = scale index within a group of
// four.  A 512-byte block of shared memory holding, for 128 rows and 4 scale
// columns, row r's 4 scales at byte (r % 32) * 16 + (r / 32) * 4 becomes
// exactly that group through one tcgen05.cp 32x128b.warpx4 (32 lanes x 16
// bytes, copied into all four lane quarters).  kq_sf_tile rewrites the
// row-major scale bytes into such 512-byte blocks once per operand.
//
// Two kernels.  When M and K are multiples of 256 and N of 192 or 256, a
// cluster of two CTAs computes 256 x 192 or 256 x 256 tiles with the pair MMA
// (gemm_pair_kernel, below).  Otherwise the single-CTA kernel described here
// runs.
//
// Tiling.  Y is cut into 128 x 128 tiles; persistent CTAs (two per SM) walk
// them.  Within a tile K advances in steps of 128
// (64 bytes of codes per row, 4 scales): per step one TMA load of A and of B
// (128 rows x 64 bytes, 64-byte swizzle: the canonical K-major operand
// layout), one bulk copy of each 512-byte scale block, two MMAs of K = 64.
// Roles (192 threads): warp 0 lane 0 loads (S stages), warp 1 owns tensor
// memory and lane 0 issues the scale copies and MMAs, warps 2..5 read the
// accumulator (one row per thread) 32 columns at a time and stage each
// 128 x 32 fp32 slice in shared memory (128-byte swizzle) for a TMA tensor
// store (when N is a multiple of 4; otherwise they store rows directly).  Every wait is
// bounded; a wait that runs out sets the device status word and the CTA
// drains and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "kq.h"
#include "kq_device.cuh"
#include "kq_host.h"

namespace kq {
namespace gemm {

constexpr int kThreads = 192;
constexpr int kTile = 128;          // M and N of the CTA tile (and of the MMA)
constexpr int kKStep = 128;         // K per stage (fp4 elements)
constexpr int kStages = 5;
constexpr int kOpBytes = kTile * kKStep / 2;        // 8 KiB of codes per operand per stage
constexpr int kSfBytes = 512;
constexpr int kStageBytes = 2 * kOpBytes + 2 * kSfBytes;
constexpr int kChunkBytes = kTile * 128;           // one 128-row x 32-column fp32 slice of Y
constexpr int kStagesBf16 = 4;                     // bf16 Y: the whole tile is staged (32 KiB)
constexpr int kTileBf16Bytes = kTile * kTile * 2;

// Dynamic shared memory of one CTA (stages, Y staging, barriers).
__host__ __device__ constexpr int smem_bytes(bool bf16) {
  return 1024 + (bf16 ? kStagesBf16 : kStages) * kStageBytes + (bf16 ? kTileBf16Bytes : kChunkBytes) + 256;
}
constexpr int kEpiThreads = 128;
constexpr int kTmemCols = 256;      // 128 accumulator columns + 8 scale columns
constexpr int kSfaCol = 128, kSfbCol = 132;

// Block-scaled instruction descriptor: A, B = E2M1 (MXF4), scales E8M0,
// both K-major, N = 128, M = 128, K = 64; the scale-factor ids go in bits
// 29-30 (A) and 4-5 (B).
constexpr uint32_t kIdescBase = (1u << 7) | (1u << 10) | ((uint32_t)(kTile >> 3) << 17) | (1u << 23) |
                                ((uint32_t)(kTile >> 4) << 24);

__device__ __forceinline__ uint64_t sw64_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(512 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)4 << 61);
}

// Descriptor of one 512-byte scale block as the source of tcgen05.cp:
// 32 rows of 16 bytes, no swizzle, 8-row groups 128 bytes apart.
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)(128 >> 4) << 32) | ((uint64_t)1 << 46);
}

__device__ __forceinline__ void mma_mxf4(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t sfa, uint32_t sfb, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(accum), "r"(sfa), "r"(sfb)
      : "memory");
}

__device__ __forceinline__ void sf_copy(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
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

__device__ __forceinline__ void tma_store_2d(const void* tmap, int c0, int c1, uint32_t src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
               ::"l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void epi_barrier(int threads = kEpiThreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(threads) : "memory");
}
// Barrier 1 among the epilogue warps that also ORs a flag across them, so
// that all of them take the same branch (none is left at a barrier).
__device__ __forceinline__ bool epi_any(bool pred, int threads = kEpiThreads) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(threads)
      : "memory");
  return r != 0;
}

// 1-D bulk copy global -> shared, completion on an mbarrier (16-byte aligned).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
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
}

// 32 consecutive fp32 accumulator columns of this thread's lane; the
// registers are valid only after tmem_wait_ld().
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20,"
      "%21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

struct GemmArgs {
  int M, N, K;
  int k_steps;               // K / 128
  const uint8_t* sfa;        // blocked scales of A: [ceil(M/128)][K/128][512]
  const uint8_t* sfb;        // blocked scales of B
  int m_tiles, n_tiles;
  void* Y;                   // [M][N] fp32, or bf16 in the bf16 variant
  const float* mu;           // optional rank-1 term: Y += mu wsum^T (mu [M], wsum [N])
  const float* wsum;
  int tma_store;             // 1: Y leaves through shared memory and TMA stores (N % 4 == 0)
};

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Persistent: CTA b takes tiles b, b + G, b + 2G, ... (tile t = (t % m_tiles,
// t / m_tiles), so CTAs running together share B tiles in L2).  The stage
// ring runs on across tiles, and the accumulator is handed back to the MMA
// lane as soon as the epilogue has read it, so the next tile's loads and MMAs
// overlap this tile's stores; two CTAs share an SM.  kRank1: the epilogue adds
// mu[m] * wsum[n] (kq_gemm_mxfp4_rank1); a compile-time switch, so that the
// plain GEMM's epilogue keeps its registers.  kBf16: Y is bf16
// (kq_gemm_mxfp4_bf16); the epilogue then stages the whole 128 x 128 tile
// (32 KiB), hands the accumulator back as soon as it has been read, and the
// tile leaves by two TMA stores while the next tile's MMAs run.
template <bool kRank1, bool kBf16>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
            const __grid_constant__ CUtensorMap ymap, const GemmArgs args, unsigned int* devstat) {
  constexpr int kS = kBf16 ? kStagesBf16 : kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  // fp32: one [128 rows][128 B] slice; bf16: two [128 rows][128 B] halves of the tile
  uint8_t* out_chunk = smem + kS * kStageBytes;                    // 128B swizzle
  uint64_t* bars = reinterpret_cast<uint64_t*>(out_chunk + (kBf16 ? kTileBf16Bytes : kChunkBytes));
  const uint32_t full0 = smem_addr(&bars[0]), empty0 = smem_addr(&bars[kS]);
  const uint32_t accf = smem_addr(&bars[2 * kS]), acce = smem_addr(&bars[2 * kS + 1]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&bars[2 * kS + 2]);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[2 * kS + 3]);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KS = args.k_steps;
  const int n_tiles_total = args.m_tiles * args.n_tiles;
  const int my_tiles = (int)blockIdx.x < n_tiles_total
                           ? (n_tiles_total - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x
                           : 0;

  pdl_launch_dependents();
  if (tid == 0) {
    tma_prefetch_desc(&amap);
    tma_prefetch_desc(&bmap);
    if (args.tma_store) tma_prefetch_desc(&ymap);
    for (int s = 0; s < kS; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(accf, 1);
    mbar_init(acce, kEpiThreads / 32);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_wait_predecessor();
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0, seq = 0;
      for (int i = 0; i < my_tiles && !*abort_flag; ++i) {
        const int t = (int)blockIdx.x + i * (int)gridDim.x;
        const int m_tile = t % args.m_tiles, n_tile = t / args.m_tiles;
        const uint8_t* sfa_tile = args.sfa + (size_t)m_tile * KS * kSfBytes;
        const uint8_t* sfb_tile = args.sfb + (size_t)n_tile * KS * kSfBytes;
        for (int kt = 0; kt < KS; ++kt, ++seq) {
          const int s = seq % kS;
          if (seq >= kS && !mbar_wait_bounded(empty0 + 8 * s, (uint32_t)(seq / kS - 1) & 1u)) {
            *abort_flag = 1;
            atomicOr(devstat, (unsigned)KQ_DEVSTAT_WAIT_TIMEOUT);
            break;
          }
          if (*abort_flag) break;
          uint8_t* st = smem + s * kStageBytes;
          const uint32_t bar = full0 + 8 * s;
          mbar_arrive_expect_tx(bar, (uint32_t)kStageBytes);
          tma_load_2d(smem_addr(st), &amap, kt * (kKStep / 2), m_tile * kTile, bar);
          tma_load_2d(smem_addr(st + kOpBytes), &bmap, kt * (kKStep / 2), n_tile * kTile, bar);
          bulk_load(smem_addr(st + 2 * kOpBytes), sfa_tile + (size_t)kt * kSfBytes, kSfBytes, bar);
          bulk_load(smem_addr(st + 2 * kOpBytes + kSfBytes), sfb_tile + (size_t)kt * kSfBytes, kSfBytes, bar);
          issued = seq + 1;
        }
      }
      if (*abort_flag) {
        const int lo = issued > kS ? issued - kS : 0;
        for (int q = lo; q < issued; ++q)
          (void)mbar_wait_bounded(full0 + 8 * (q % kS), (uint32_t)(q / kS) & 1u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int seq = 0;
      bool issued_any = false;
      for (int i = 0; i < my_tiles; ++i) {
        // the epilogue has read the previous tile's accumulator
        bool ok = i == 0 || mbar_wait_bounded(acce, (uint32_t)(i - 1) & 1u);
        if (ok) fence_after_sync();
        for (int kt = 0; ok && kt < KS; ++kt, ++seq) {
          const int s = seq % kS;
          ok = mbar_wait_bounded(full0 + 8 * s, (uint32_t)(seq / kS) & 1u) && !*abort_flag;
          if (!ok) break;
          fence_after_sync();
          const uint32_t st = smem_addr(smem + s * kStageBytes);
          // scale blocks of this step into tensor memory (in issue order with
          // the MMAs below, and after the MMAs of the previous step)
          sf_copy(tmem_base + kSfaCol, sf_desc(st + 2 * kOpBytes));
          sf_copy(tmem_base + kSfbCol, sf_desc(st + 2 * kOpBytes + kSfBytes));
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const uint32_t sf_id = (uint32_t)(2 * kk);      // scales 2kk, 2kk+1 of the group of 4
            const uint32_t sfa = (tmem_base + kSfaCol) | (sf_id << 30);
            const uint32_t sfb = (tmem_base + kSfbCol) | (sf_id << 30);
            const uint32_t idesc = kIdescBase | (sf_id << 29) | (sf_id << 4);
            mma_mxf4(tmem_base, sw64_desc(st + kk * 32), sw64_desc(st + kOpBytes + kk * 32), idesc,
                     sfa, sfb, (kt | kk) != 0);
          }
          mma_commit(empty0 + 8 * s);
          issued_any = true;
        }
        if (!ok) {
          *abort_flag = 1;
          atomicOr(devstat, (unsigned)KQ_DEVSTAT_WAIT_TIMEOUT);
          break;
        }
        mma_commit(accf);
      }
      if (*abort_flag && issued_any) {
        // give the MMAs already issued (microseconds of work) time to finish
        // before tensor memory is freed
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 20000000ull) {}
      }
    }
  } else {
    // epilogue: warps 2..5 -> TMEM lane quarters (warp % 4); thread = one row
    if constexpr (kBf16) {
      const int q = warp & 3;
      const int etid = tid - 64;
      const int r_local = 32 * q + lane;
      for (int i = 0; i < my_tiles; ++i) {
        const int t = (int)blockIdx.x + i * (int)gridDim.x;
        const int m_tile = t % args.m_tiles, n_tile = t / args.m_tiles;
        const int row = m_tile * kTile + r_local;
        const bool ok = mbar_wait_bounded(accf, (uint32_t)i & 1u);
        // the previous tile's stores have read the staging buffer
        if (args.tma_store && etid == 0) bulk_wait_read_all();
        if (epi_any(!ok || *abort_flag)) {
          if (!ok) atomicOr(devstat, (unsigned)KQ_DEVSTAT_WAIT_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        fence_after_sync();
        const int n0 = n_tile * kTile;
        for (int c = 0; c < kTile / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(32 * c), r);
          uint32_t w[16];                  // bf16 pairs, even column in the low half
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1]));
            w[k] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          if (c == kTile / 32 - 1) {
            // the whole accumulator is in registers or staged: hand it back
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(acce);
          }
          if (args.tma_store) {
            // half c / 2 of the tile: [128 rows][64 columns = 128 B], 16-byte
            // chunk j of a row at (j ^ (row % 8)) * 16 (128-byte swizzle)
            uint8_t* rowp = out_chunk + (c >> 1) * (kTile * 128) + r_local * 128;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int j = (c & 1) * 4 + u;
              *reinterpret_cast<uint4*>(rowp + ((j ^ (r_local & 7)) << 4)) =
                  make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
            }
          } else if (row < args.M) {
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(args.Y) + (size_t)row * args.N + n0 + 32 * c;
            const int n_valid = args.N - (n0 + 32 * c);
            const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(w);
            for (int k = 0; k < 32 && k < n_valid; ++k) dst[k] = src[k];
          }
        }
        if (args.tma_store) {
          // generic-proxy writes -> visible to the TMA stores, then all warps done
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          epi_barrier();
          if (etid == 0) {
            tma_store_2d(&ymap, n0, m_tile * kTile, smem_addr(out_chunk));
            tma_store_2d(&ymap, n0 + 64, m_tile * kTile, smem_addr(out_chunk + kTile * 128));
            bulk_commit();
          }
        }
      }
      if (args.tma_store && etid == 0) bulk_wait_all();
    } else {
      const int q = warp & 3;
      const int etid = tid - 64;
      const int r_local = 32 * q + lane;
      for (int i = 0; i < my_tiles; ++i) {
        const int t = (int)blockIdx.x + i * (int)gridDim.x;
        const int m_tile = t % args.m_tiles, n_tile = t / args.m_tiles;
        const int row = m_tile * kTile + r_local;
        const bool ok = mbar_wait_bounded(accf, (uint32_t)i & 1u);
        if (epi_any(!ok || *abort_flag)) {
          if (!ok) atomicOr(devstat, (unsigned)KQ_DEVSTAT_WAIT_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        fence_after_sync();
        const int n0 = n_tile * kTile;
        for (int c = 0; c < kTile / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(32 * c), r);
          if constexpr (kRank1) {
            // the centring variant's removed mean, restored in fp32
            const float m = row < args.M ? args.mu[row] : 0.0f;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              const int col = n0 + 32 * c + k;
              const float ws = col < args.N ? __ldg(args.wsum + col) : 0.0f;
              r[k] = __float_as_uint(__fmaf_rn(m, ws, __uint_as_float(r[k])));
            }
          }
          if (c == kTile / 32 - 1) {
            // the whole accumulator is in registers or staged: hand it back
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(acce);
          }
          if (args.tma_store) {
            // the previous slice's store has read the staging chunk
            if (etid == 0) bulk_wait_read_all();
            epi_barrier();
            uint8_t* rowp = out_chunk + r_local * 128;
#pragma unroll
            for (int u = 0; u < 8; ++u)
              *reinterpret_cast<uint4*>(rowp + ((u ^ (r_local & 7)) << 4)) =
                  make_uint4(r[4 * u], r[4 * u + 1], r[4 * u + 2], r[4 * u + 3]);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            epi_barrier();
            if (etid == 0) {
              tma_store_2d(&ymap, n0 + 32 * c, m_tile * kTile, smem_addr(out_chunk));
              bulk_commit();
            }
          } else if (row < args.M) {
            float* dst = static_cast<float*>(args.Y) + (size_t)row * args.N + n0 + 32 * c;
            const int n_valid = args.N - (n0 + 32 * c);
            for (int k = 0; k < 32 && k < n_valid; ++k) dst[k] = __uint_as_float(r[k]);
          }
        }
      }
      if (args.tma_store && etid == 0) bulk_wait_all();
    }
  }

  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// CTA-pair kernel: 256 x kTN output tiles over two SMs (cta_group::2)
// ---------------------------------------------------------------------------
// A cluster of two CTAs on two SMs computes one 256 x kTN tile of Y at a
// time with the pair form of the block-scaled MMA: CTA r (r = 0, 1) holds rows
// 128 r .. 128 r + 127 of the A tile and rows r kTN/2 .. (r + 1) kTN/2 - 1 of
// the B tile in its own shared memory, and each MMA (issued by CTA 0) reads A
// from both CTAs and B from both CTAs, leaving rows 128 r .. of the 256 x kTN
// product in CTA r's tensor memory.  Every byte of A and B therefore crosses
// from L2 once per pair instead of once per 128-row tile: half the operand
// traffic of the single-CTA kernel per FLOP.  The scales of a CTA's A rows and
// of the B rows of the tile are staged in each CTA and moved into its own
// tensor memory by the pair copy.  No load uses cluster multicast: each CTA
// loads only into its own shared memory; the loads of both CTAs complete on
// CTA 0's barrier, and CTA 0's MMA completions arrive on both CTAs' barriers.
//
// Tile width.  kTN = 256 (N a multiple of 256): one accumulator of 256
// columns (two would leave no column for the scales), handed back as soon as
// the epilogue has read it, before the stores.  kTN = 192 (N a multiple of
// 192 but not of 256): two accumulators of 192 columns fit beside the scales,
// so the MMAs of the next tile run while the epilogue drains the last one;
// where both widths apply the 256-wide tile wins, since the 192-wide one loads
// 17 % more operand bytes per FLOP and the operand stream bounds the
// mainloop.  Scale blocks cover 128 B rows; a 192-column tile with an odd
// index starts half-way through one, so it loads the two blocks it meets and
// points the MMA's B-scale address two tensor-memory columns (64 rows) in.
//
// A stage holds K = 256 (128-byte rows, 128-byte swizzle): per stage one
// barrier round trip, six scale copies and four MMAs of K = 64.  With 64-byte
// rows (K = 128, two MMAs a stage) the same kernel ran the 4608 x 3072 x 12288
// layer no faster than the single-CTA kernel (117 against 108 us): the issue
// of each stage, not operand bandwidth, was the limit.
//
// Roles (320 threads per CTA): warp 0 lane 0 loads (in both CTAs), warp 1
// owns tensor memory (both CTAs) and, in CTA 0, lane 0 issues the scale
// copies and the MMAs; warps 2..9 read the accumulator (two warps per lane
// quarter, one row per thread, half of the columns each, in one round trip),
// hand it back, stage Y in shared memory and write it with TMA tensor stores.
// Every wait is bounded; a wait that runs out sets the device status word,
// the CTA drains, meets its peer at the final cluster barrier and exits.
constexpr int kPM = 256;                           // tile rows of a pair (the MMA's M)
constexpr int kPHalf = 128;                        // rows of A in each CTA
constexpr int kPK = 256;                           // K per stage (fp4 elements): 128-byte rows
constexpr int kPKb = kPK / 128;                    // 128-K scale blocks per stage
constexpr int kPOpBytes = kPHalf * kPK / 2;        // A codes per CTA per stage
constexpr int kPTmemCols = 512;
constexpr int kPAccStride = 256;                   // tensor-memory columns between accumulators

template <int kTN>
struct PairShape {
  static_assert(kTN == 192 || kTN == 256, "pair tile width");
  static constexpr int kBHalf = kTN / 2;                        // rows of B in each CTA
  static constexpr int kBufs = kTN == 256 ? 1 : 2;              // accumulators
  static constexpr int kStages = 5;
  // [128 rows][128 B] staging chunks: two for 256-wide tiles (Y leaves in
  // rounds of two chunks; the stages take the rest of shared memory)
  static constexpr int kOutChunks = kTN == 256 ? 2 : 4;
  static constexpr int kBBytes = kBHalf * kPK / 2;              // B codes per CTA per stage
  // bytes one CTA loads per stage: codes, A's scale blocks, two blocks of B scales
  static constexpr int kStageTx = kPOpBytes + kBBytes + 3 * kPKb * kSfBytes;
  static constexpr int kStageBytes = (kStageTx + 1023) & ~1023;   // a multiple of 1 KiB
  // after the accumulators: A scales (4 columns per 128-K block), then B
  // scales (8 columns per 128-K block: two 128-row blocks)
  static constexpr int kSfaCol = (kBufs - 1) * kPAccStride + kTN;
  static constexpr int kSfbCol = kSfaCol + 4 * kPKb;
  static_assert(kSfbCol + 8 * kPKb <= kPTmemCols, "tensor memory layout");
  // M = 256 (the pair), N = kTN, K = 64, E2M1 x E2M1, E8M0 scales, K-major
  static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(kTN >> 3) << 17) | (1u << 23) |
                                     ((uint32_t)(kPM >> 4) << 24);
  static constexpr int kSmem = 1024 + kStages * kStageBytes + kOutChunks * kPHalf * 128 + 256;
  static_assert(kSmem <= 232448, "shared memory per CTA");
};

// Shared-memory descriptor of a K-major operand tile whose rows are 128 bytes
// (K = 256 fp4), 128-byte swizzle: 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

// Arrive on an mbarrier of another CTA of the cluster (release at cluster scope).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

// 2-D TMA load into this CTA's shared memory whose completion is counted on a
// barrier of CTA 0 of the pair (`bar` is that barrier's cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void* tmap, int c0, int c1,
                                                 uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void mma_mxf4_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                              uint32_t sfa, uint32_t sfb, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(accum), "r"(sfa), "r"(sfb)
      : "memory");
}

// Scale block from each CTA's shared memory into its own tensor memory.
__device__ __forceinline__ void sf_copy_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Arrive on the barrier at this offset in both CTAs of the pair once the
// MMAs issued so far have completed.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\t"
      "mov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}"
      ::"r"(bar)
      : "memory");
}

constexpr int kPEpiWarps = 8;                      // two per tensor-memory lane quarter
constexpr int kPEpiThreads = 32 * kPEpiWarps;
constexpr int kPThreads = 64 + kPEpiThreads;

struct PairArgs {
  int M, N;
  int k_steps;               // stages of K per tile (K / 256)
  int m_tiles, n_tiles;      // 256-row and kTN-column tiles
  int pairs;                 // clusters in the grid
};

// Bounded wait for a time well above any in-flight copy or MMA, used only on
// the abort path before the CTA leaves (nothing else tells it when the
// peer's copies into its shared memory have landed).
__device__ __forceinline__ void settle_ns(uint64_t ns) {
  const uint64_t t0 = global_timer_ns();
  while (global_timer_ns() - t0 < ns) {}
}

template <bool kBf16, int kTN>
__global__ void __launch_bounds__(kPThreads, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                 const __grid_constant__ CUtensorMap sfamap, const __grid_constant__ CUtensorMap sfbmap,
                 const __grid_constant__ CUtensorMap ymap, const PairArgs args, unsigned int* devstat) {
  using P = PairShape<kTN>;
  constexpr int kS = P::kStages, kB = P::kBufs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* out_stage = smem + kS * P::kStageBytes;                // [128 rows][128 B] chunks, 128B swizzle
  uint64_t* bars = reinterpret_cast<uint64_t*>(out_stage + P::kOutChunks * kPHalf * 128);
  const uint32_t full0 = smem_addr(&bars[0]), empty0 = smem_addr(&bars[kS]);
  const uint32_t accf0 = smem_addr(&bars[2 * kS]), acce0 = smem_addr(&bars[2 * kS + kB]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&bars[2 * kS + 2 * kB]);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[2 * kS + 2 * kB + 1]);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();              // 0: issues the MMAs
  const int pair = (int)blockIdx.x >> 1;
  const int KS = args.k_steps;             // stages of K per tile
  const int KS128 = KS * kPKb;             // 128-K scale blocks per row block
  const int n_tiles_total = args.m_tiles * args.n_tiles;
  const int my_tiles = pair < n_tiles_total ? (n_tiles_total - pair + args.pairs - 1) / args.pairs : 0;

  pdl_launch_dependents();
  if (tid == 0) {
    tma_prefetch_desc(&amap);
    tma_prefetch_desc(&bmap);
    tma_prefetch_desc(&sfamap);
    tma_prefetch_desc(&sfbmap);
    tma_prefetch_desc(&ymap);
    for (int s = 0; s < kS; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < kB; ++b) {
      mbar_init(accf0 + 8 * b, 1);
      mbar_init(acce0 + 8 * b, 2 * kPEpiWarps);           // every epilogue warp of both CTAs
    }
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(kPTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  fence_before_sync();
  // both CTAs' barriers are initialised before any copy or commit targets them
  cluster_sync_all();
  fence_after_sync();
  pdl_wait_predecessor();
  const uint32_t tmem_base = *tmem_slot;
  bool aborted = false;

  if (warp == 0) {
    if (lane == 0) {
      int seq = 0;
      for (int i = 0; i < my_tiles && !*abort_flag; ++i) {
        const int t = pair + i * args.pairs;
        const int m_tile = t % args.m_tiles, n_tile = t / args.m_tiles;
        const int arow = m_tile * kPM + (int)rank * kPHalf;
        const int bcol0 = n_tile * kTN;
        const int brow = bcol0 + (int)rank * P::kBHalf;
        // the 128-row scale blocks of A's rows of this CTA, and the first of
        // the two that the tile's B rows meet
        const int sfa_blk = (m_tile * 2 + (int)rank) * KS128, sfb_blk = (bcol0 >> 7) * KS128;
        for (int kt = 0; kt < KS; ++kt, ++seq) {
          const int s = seq % kS;
          if (seq >= kS && !mbar_wait_bounded(empty0 + 8 * s, (uint32_t)(seq / kS - 1) & 1u)) {
            *abort_flag = 1;
            atomicOr(devstat, (unsigned)KQ_DEVSTAT_WAIT_TIMEOUT);
            break;
          }
          const uint32_t st = smem_addr(smem + s * P::kStageBytes);
          const uint32_t bar = map_to_rank(full0 + 8 * s, 0);
          if (rank == 0) mbar_arrive_expect_tx(full0 + 8 * s, (uint32_t)(2 * P::kStageTx));
          // codes, then the scale blocks of this stage's kPKb 128-K blocks: A's
          // rows, then the two 128-row blocks of B
          tma_load_2d_pair(st, &amap, kt * (kPK / 2), arow, bar);
          tma_load_2d_pair(st + kPOpBytes, &bmap, kt * (kPK / 2), brow, bar);
          const uint32_t sf = st + kPOpBytes + P::kBBytes;
          tma_load_2d_pair(sf, &sfamap, 0, sfa_blk + kPKb * kt, bar);
          tma_load_2d_pair(sf + kPKb * kSfBytes, &sfbmap, 0, sfb_blk + kPKb * kt, bar);
          tma_load_2d_pair(sf + 2 * kPKb * kSfBytes, &sfbmap, 0, sfb_blk + KS128 + kPKb * kt, bar);
        }
      }
      aborted = *abort_flag != 0;
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      int seq = 0;
      for (int i = 0; i < my_tiles; ++i) {
        const int buf = i % kB, use = i / kB;
        const int n_tile = (pair + i * args.pairs) / args.m_tiles;
        // B scale of tile row 0 sits at row (n_tile kTN) % 128 of its block:
        // 32 rows per tensor-memory column
        const uint32_t sfb_shift = (uint32_t)(((n_tile * kTN) & 127) >> 5);
        const uint32_t acc = tmem_base + (uint32_t)(buf * kPAccStride);
        // both CTAs' epilogues have read this accumulator's previous tile
        bool ok = use == 0 || mbar_wait_bounded(acce0 + 8 * buf, (uint32_t)(use - 1) & 1u);
        if (ok) fence_after_sync();
        for (int kt = 0; ok && kt < KS; ++kt, ++seq) {
          const int s = seq % kS;
          ok = mbar_wait_bounded(full0 + 8 * s, (uint32_t)(seq / kS) & 1u) && !*abort_flag;
          if (!ok) break;
          fence_after_sync();
          const uint32_t st = smem_addr(smem + s * P::kStageBytes);
          const uint32_t sf = st + kPOpBytes + P::kBBytes;
#pragma unroll
          for (int j = 0; j < kPKb; ++j) {
            sf_copy_pair(tmem_base + P::kSfaCol + 4 * j, sf_desc(sf + j * kSfBytes));
            sf_copy_pair(tmem_base + P::kSfbCol + 8 * j, sf_desc(sf + (kPKb + j) * kSfBytes));
            sf_copy_pair(tmem_base + P::kSfbCol + 8 * j + 4, sf_desc(sf + (2 * kPKb + j) * kSfBytes));
          }
          // K = 64 per MMA: MMA kk reads scale block kk / 2, scales 2 (kk % 2) and 2 (kk % 2) + 1
#pragma unroll
          for (int kk = 0; kk < 2 * kPKb; ++kk) {
            const int j = kk >> 1;
            const uint32_t sf_id = (uint32_t)(2 * (kk & 1));
            const uint32_t sfa = (tmem_base + P::kSfaCol + 4 * j) | (sf_id << 30);
            const uint32_t sfb = (tmem_base + P::kSfbCol + 8 * j + sfb_shift) | (sf_id << 30);
            const uint32_t idesc = P::kIdesc | (sf_id << 29) | (sf_id << 4);
            mma_mxf4_pair(acc, sw128_desc(st + kk * 32), sw128_desc(st + kPOpBytes + kk * 32), idesc, sfa,
                          sfb, (kt | kk) != 0);
          }
          mma_commit_pair(empty0 + 8 * s);
        }
        if (!ok) {
          *abort_flag = 1;
          atomicOr(devstat, (unsigned)KQ_DEVSTAT_WAIT_TIMEOUT);
          break;
        }
        mma_commit_pair(accf0 + 8 * buf);
      }
      aborted = *abort_flag != 0;
    }
  } else {
    // epilogue: warps 2 .. 2 + kPEpiWarps - 1.  Warp w reads tensor-memory
    // lane quarter w % 4 (32 rows, one per thread) and half (w - 2) / 4 of
    // the tile's columns in one round trip, hands the accumulator back, then
    // stages Y in shared memory and writes it with TMA tensor stores.
    constexpr int kHalfCols = kTN / 2;
    constexpr int kCC = kBf16 ? 64 : 32;       // Y columns per staging chunk (128 bytes a row)
    constexpr int kChunks = kTN / kCC;
    constexpr int kW = kBf16 ? 8 : 4;          // Y columns per 16-byte group
    const int q = warp & 3, h = (warp - 2) >> 2;
    const int etid = tid - 64;
    const int r_local = 32 * q + lane;
    const int col0 = h * kHalfCols;
    for (int i = 0; i < my_tiles; ++i) {
      const int buf = i % kB, use = i / kB;
      const int t = pair + i * args.pairs;
      const int m_tile = t % args.m_tiles, n_tile = t / args.m_tiles;
      const int row0 = m_tile * kPM + (int)rank * kPHalf, n0 = n_tile * kTN;
      const bool ok = mbar_wait_bounded(accf0 + 8 * buf, (uint32_t)use & 1u);
      // the previous tile's stores have read the staging chunks
      if (etid == 0) bulk_wait_read_all();
      if (epi_any(!ok || *abort_flag, kPEpiThreads)) {
        if (!ok) atomicOr(devstat, (unsigned)KQ_DEVSTAT_WAIT_TIMEOUT);
        *abort_flag = 1;
        aborted = true;
        break;
      }
      fence_after_sync();
      const uint32_t acc = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * kPAccStride + col0);
      // 32-column loads (each starts at a multiple of 32 columns), one wait
      uint32_t v[kHalfCols / 32][32];
#pragma unroll
      for (int g = 0; g < kHalfCols / 32; ++g) tmem_ld32_nowait(acc + 32 * g, v[g]);
      tmem_wait_ld();
      // keep every use of the loaded registers after the wait
#pragma unroll
      for (int g = 0; g < kHalfCols / 32; ++g)
#pragma unroll
        for (int k = 0; k < 32; ++k) asm volatile("" : "+r"(v[g][k]));
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(map_to_rank(acce0 + 8 * buf, 0));
      // Four 16-byte words of Y (columns a .. a + 4 kW / 4 - 1 of this warp's
      // half) as they go to shared memory: fp32 bits, or bf16 pairs with the
      // even column in the low half.
      auto group = [&](int a, uint32_t (&w)[4]) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if constexpr (kBf16) {
            const int b = a + 2 * e;
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(v[b >> 5][b & 31]),
                                                            __uint_as_float(v[(b + 1) >> 5][(b + 1) & 31]));
            w[e] = *reinterpret_cast<const uint32_t*>(&h2);
          } else {
            w[e] = v[(a + e) >> 5][(a + e) & 31];
          }
        }
      };
      if constexpr (kHalfCols % kCC == 0) {
        // each half is whole chunks: per round, kPer chunks of each half
        // (slots kPer h ..), so every register index is fixed at compile time
        constexpr int kHC = kHalfCols / kCC;
        constexpr int kPer = P::kOutChunks / 2;
        static_assert(P::kOutChunks % 2 == 0 && kPer >= 1, "whole staging chunks per half and round");
#pragma unroll
        for (int a = 0; a < kHC; a += kPer) {
          if (a > 0) {
            if (etid == 0) bulk_wait_read_all();
            epi_barrier(kPEpiThreads);
          }
#pragma unroll
          for (int cc = a; cc < a + kPer && cc < kHC; ++cc) {
            uint8_t* rowp = out_stage + (kPer * h + cc - a) * (kPHalf * 128) + r_local * 128;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              uint32_t w[4];
              group(cc * kCC + j * kW, w);
              *reinterpret_cast<uint4*>(rowp + ((j ^ (r_local & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          epi_barrier(kPEpiThreads);
          if (etid == 0) {
            for (int hh = 0; hh < 2; ++hh)
              for (int cc = a; cc < a + kPer && cc < kHC; ++cc)
                tma_store_2d(&ymap, n0 + hh * kHalfCols + cc * kCC, row0,
                             smem_addr(out_stage + (kPer * hh + cc - a) * (kPHalf * 128)));
            bulk_commit();
          }
        }
      } else {
        // halves split a chunk (bf16, 192 columns): chunks follow the tile,
        // and both halves write into the shared one
        static_assert(kChunks <= P::kOutChunks, "one round");
#pragma unroll
        for (int k = 0; k < kHalfCols / kW; ++k) {
          const int c = col0 + k * kW;         // first Y column of this 16-byte group
          uint32_t w[4];
          group(k * kW, w);
          const int j = (c % kCC) / kW;
          uint8_t* rowp = out_stage + (c / kCC) * (kPHalf * 128) + r_local * 128;
          *reinterpret_cast<uint4*>(rowp + ((j ^ (r_local & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        epi_barrier(kPEpiThreads);
        if (etid == 0) {
          for (int c = 0; c < kChunks; ++c)
            tma_store_2d(&ymap, n0 + c * kCC, row0, smem_addr(out_stage + c * (kPHalf * 128)));
          bulk_commit();
        }
      }
    }
    if (etid == 0) bulk_wait_all();
  }

  // Leave together: after a timeout, give copies and MMAs already in flight
  // (microseconds of work) time to land first; then every thread of both
  // CTAs meets at the cluster barrier, so no CTA exits while its peer may
  // still reach its shared or tensor memory.
  if (__syncthreads_or(aborted)) settle_ns(20000000ull);
  fence_before_sync();
  cluster_sync_all();
  if (warp == 1) {
    fence_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kPTmemCols)
                 : "memory");
  }
}

// Row-major scale bytes [R][K/32] -> 512-byte blocks [ceil(R/128)][K/128][512]
// (row r, scale column s at byte (r % 32) * 16 + ((r % 128) / 32) * 4 + s % 4
// of block (r / 128, s / 4)); rows past R become zero.  One thread per output byte.
__global__ void __launch_bounds__(256)
sf_tile_kernel(const uint8_t* __restrict__ scales, int R, int ns, int n_out, uint8_t* __restrict__ out) {
  for (int o = blockIdx.x * blockDim.x + threadIdx.x; o < n_out; o += gridDim.x * blockDim.x) {
    const int blk = o >> 9, within = o & 511;
    const int groups = ns >> 2;
    const int rt = blk / groups, g = blk - rt * groups;
    const int r0 = within >> 4, r1 = (within >> 2) & 3, j = within & 3;
    const int r = rt * 128 + r1 * 32 + r0;
    out[o] = r < R ? scales[(size_t)r * ns + 4 * g + j] : (uint8_t)0;
  }
}

}  // namespace gemm

namespace {

PFN_cuTensorMapEncodeTiled_v12000 gemm_encoder() {
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

int codes_tmap(CUtensorMap* tm, const uint8_t* codes, int64_t rows, int64_t K) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = gemm_encoder();
  if (!enc) return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled not found in the CUDA driver");
  const cuuint64_t dims[2] = {(cuuint64_t)K / 2, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)K / 2};
  const cuuint32_t box[2] = {gemm::kKStep / 2, gemm::kTile};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides,
                         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return KQ_OK;
}

constexpr int kMaxDevices = 64;

// Tiled scale blocks [rows / 128 * K / 128][512 bytes] seen as a 2-D tensor of
// 128 32-bit words per block; one box is one 512-byte block.
int sf_tmap(CUtensorMap* tm, const uint8_t* tiled, int64_t rows, int64_t K) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = gemm_encoder();
  if (!enc) return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled not found in the CUDA driver");
  const cuuint64_t dims[2] = {128, (cuuint64_t)((rows + 127) / 128 * (K / 128))};
  const cuuint64_t strides[1] = {512};
  const cuuint32_t box[2] = {128, (cuuint32_t)gemm::kPKb};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint8_t*>(tiled), dims, strides,
                         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled (scales) failed (CUresult %d)", (int)r);
  return KQ_OK;
}

// Codes [rows][K/2] for the pair kernel: box 128 bytes (K = 256) x box_rows
// rows, 128-byte swizzle (the canonical K-major layout of 128-byte rows).
int pair_codes_tmap(CUtensorMap* tm, const uint8_t* codes, int64_t rows, int64_t K, int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = gemm_encoder();
  if (!enc) return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled not found in the CUDA driver");
  const cuuint64_t dims[2] = {(cuuint64_t)K / 2, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)K / 2};
  const cuuint32_t box[2] = {gemm::kPK / 2, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides,
                         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return KQ_OK;
}

// The CTA-pair kernel with kTN-column tiles, for M a multiple of 256, N of
// kTN and K of the stage's K (no rank-1 term).
template <int kTN>
int gemm_pair_launch(const uint8_t* a_codes, const uint8_t* b_codes, const CUtensorMap& ym,
                     const uint8_t* a_sf_tiled, const uint8_t* b_sf_tiled, int64_t M, int64_t N,
                     int64_t K, bool bf16, unsigned int* devstat, cudaStream_t stream) {
  using P = gemm::PairShape<kTN>;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return cuda_fail(err, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(KQ_ERR_UNSUPPORTED, "device ordinal %d", dev);
  const int smem = P::kSmem;
  static std::once_flag attr_once[kMaxDevices];
  static cudaError_t attr_err[kMaxDevices];
  std::call_once(attr_once[dev], [&] {
    attr_err[dev] = cudaFuncSetAttribute(gemm::gemm_pair_kernel<false, kTN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (attr_err[dev] == cudaSuccess)
      attr_err[dev] = cudaFuncSetAttribute(gemm::gemm_pair_kernel<true, kTN>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (attr_err[dev] != cudaSuccess) return cuda_fail(attr_err[dev], "cudaFuncSetAttribute (pair)");

  CUtensorMap am, bm, sam, sbm;
  if (int st = pair_codes_tmap(&am, a_codes, M, K, gemm::kPHalf)) return st;
  if (int st = pair_codes_tmap(&bm, b_codes, N, K, P::kBHalf)) return st;
  if (int st = sf_tmap(&sam, a_sf_tiled, M, K)) return st;
  if (int st = sf_tmap(&sbm, b_sf_tiled, N, K)) return st;
  gemm::PairArgs args;
  args.M = (int)M;
  args.N = (int)N;
  args.k_steps = (int)(K / gemm::kPK);
  args.m_tiles = (int)(M / gemm::kPM);
  args.n_tiles = (int)(N / kTN);

  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(gemm::kPThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  auto kern = bf16 ? gemm::gemm_pair_kernel<true, kTN> : gemm::gemm_pair_kernel<false, kTN>;
  // as many pairs as can be resident at once (one CTA per SM), no more than tiles
  int sms = 0;
  if (int st = sm_count(&sms)) return st;
  cfg.gridDim = dim3((unsigned)sms);
  int clusters = 0;
  err = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
  if (err != cudaSuccess) return cuda_fail(err, "cudaOccupancyMaxActiveClusters");
  if (clusters < 1) return fail(KQ_ERR_UNSUPPORTED, "gemm: no CTA pair fits on the device");
  const int64_t tiles = (int64_t)args.m_tiles * args.n_tiles;
  if (clusters > tiles) clusters = (int)tiles;
  args.pairs = clusters;
  cfg.gridDim = dim3((unsigned)(2 * clusters));
  err = cudaLaunchKernelEx(&cfg, kern, am, bm, sam, sbm, ym, args, devstat);
  if (err != cudaSuccess) return cuda_fail(err, "gemm_pair_kernel launch");
  return check_launch("gemm_pair_kernel launch");
}

}  // namespace
}  // namespace kq

namespace kq {

// Shared by kq_gemm_mxfp4 (mu = wsum = NULL), kq_gemm_mxfp4_rank1 and
// kq_gemm_mxfp4_bf16 (bf16: Y is bf16, no rank-1 term).
int gemm_launch(const uint8_t* a_codes, const uint8_t* a_sf_tiled, const uint8_t* b_codes,
                const uint8_t* b_sf_tiled, int64_t M, int64_t N, int64_t K, const float* mu,
                const float* wsum, void* Y, bool bf16, void* stream, const char* fn) {
  if (M < 0 || N < 0 || K <= 0 || K % 128 != 0)
    return kq::fail(KQ_ERR_INVALID_ARG, "%s: need M, N >= 0 and K a positive multiple of 128", fn);
  if (M == 0 || N == 0) return KQ_OK;
  if (!a_codes || !a_sf_tiled || !b_codes || !b_sf_tiled || !Y)
    return kq::fail(KQ_ERR_INVALID_ARG, "%s: NULL pointer", fn);
  if (!kq::aligned(a_codes, 16) || !kq::aligned(b_codes, 16) || !kq::aligned(a_sf_tiled, 16) ||
      !kq::aligned(b_sf_tiled, 16) || !kq::aligned(Y, 16))
    return kq::fail(KQ_ERR_ALIGNMENT, "%s: codes, tiled scales and Y must be 16-byte aligned", fn);
  if (M >= ((int64_t)1 << 31) || N >= ((int64_t)1 << 31) || K >= ((int64_t)1 << 24) ||
      ((M + 127) / 128) * ((N + 127) / 128) >= ((int64_t)1 << 31))
    return kq::fail(KQ_ERR_UNSUPPORTED, "%s: sizes beyond the supported range", fn);

  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return kq::cuda_fail(err, "cudaGetDevice");
  if (dev < 0 || dev >= kq::kMaxDevices) return kq::fail(KQ_ERR_UNSUPPORTED, "device ordinal %d", dev);
  const size_t smem = (size_t)kq::gemm::smem_bytes(bf16);
  static std::once_flag attr_once[kq::kMaxDevices];
  static cudaError_t attr_err[kq::kMaxDevices];
  std::call_once(attr_once[dev], [&] {
    const int s32 = kq::gemm::smem_bytes(false), s16 = kq::gemm::smem_bytes(true);
    attr_err[dev] = cudaFuncSetAttribute(kq::gemm::gemm_kernel<false, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, s32);
    if (attr_err[dev] == cudaSuccess)
      attr_err[dev] = cudaFuncSetAttribute(kq::gemm::gemm_kernel<true, false>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, s32);
    if (attr_err[dev] == cudaSuccess)
      attr_err[dev] = cudaFuncSetAttribute(kq::gemm::gemm_kernel<false, true>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, s16);
  });
  if (attr_err[dev] != cudaSuccess) return kq::cuda_fail(attr_err[dev], "cudaFuncSetAttribute");

  CUtensorMap am, bm, ym;
  if (int st = kq::codes_tmap(&am, a_codes, M, K)) return st;
  if (int st = kq::codes_tmap(&bm, b_codes, N, K)) return st;
  // TMA stores need 16-byte row strides: N a multiple of 4 (fp32) or 8 (bf16)
  const bool tma_store = (N % (bf16 ? 8 : 4)) == 0;
  memset(&ym, 0, sizeof(ym));
  if (tma_store) {
    // Y [M][N]; box 128 bytes of a row (32 fp32 or 64 bf16 columns) x 128 rows,
    // 128-byte swizzle
    PFN_cuTensorMapEncodeTiled_v12000 enc = kq::gemm_encoder();
    const cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)N * (bf16 ? 2 : 4)};
    const cuuint32_t box[2] = {bf16 ? 64u : 32u, (cuuint32_t)kq::gemm::kTile};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(&ym, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                           2, Y, dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return kq::fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled (Y) failed (CUresult %d)", (int)r);
  }
  unsigned int* devstat = nullptr;
  if (int st = kq::device_status_address(&devstat)) return st;
  if (M % kq::gemm::kPM == 0 && K % kq::gemm::kPK == 0 && mu == nullptr && tma_store) {
    if (N % 256 == 0)
      return kq::gemm_pair_launch<256>(a_codes, b_codes, ym, a_sf_tiled, b_sf_tiled, M, N, K, bf16, devstat,
                                       kq::as_stream(stream));
    if (N % 192 == 0)
      return kq::gemm_pair_launch<192>(a_codes, b_codes, ym, a_sf_tiled, b_sf_tiled, M, N, K, bf16, devstat,
                                       kq::as_stream(stream));
  }
  kq::gemm::GemmArgs args;
  args.M = (int)M;
  args.N = (int)N;
  args.K = (int)K;
  args.k_steps = (int)(K / kq::gemm::kKStep);
  args.sfa = a_sf_tiled;
  args.sfb = b_sf_tiled;
  args.Y = Y;
  args.tma_store = tma_store ? 1 : 0;
  args.m_tiles = (int)((M + 127) / 128);
  args.n_tiles = (int)((N + 127) / 128);
  args.mu = mu;
  args.wsum = wsum;

  cudaLaunchConfig_t cfg = {};
  int sms = 0;
  if (int st = kq::sm_count(&sms)) return st;
  const int64_t tiles = (int64_t)args.m_tiles * args.n_tiles;
  const int64_t slots = 2 * (int64_t)sms;                    // two CTAs per SM
  cfg.gridDim = dim3((unsigned)(tiles < slots ? tiles : slots));
  cfg.blockDim = dim3(kq::gemm::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = kq::as_stream(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (bf16)
    err = cudaLaunchKernelEx(&cfg, kq::gemm::gemm_kernel<false, true>, am, bm, ym, args, devstat);
  else if (mu != nullptr)
    err = cudaLaunchKernelEx(&cfg, kq::gemm::gemm_kernel<true, false>, am, bm, ym, args, devstat);
  else
    err = cudaLaunchKernelEx(&cfg, kq::gemm::gemm_kernel<false, false>, am, bm, ym, args, devstat);
  if (err != cudaSuccess) return kq::cuda_fail(err, "gemm_kernel launch");
  return kq::check_launch("gemm_kernel launch");
}

}  // namespace kq

extern "C" {

int kq_sf_tile(const uint8_t* scales, int64_t R, int64_t K, uint8_t* tiled, void* stream) {
  const char* fn = "kq_sf_tile";
  if (R < 0 || K <= 0 || K % 128 != 0)
    return kq::fail(KQ_ERR_INVALID_ARG, "%s: need R >= 0 and K a positive multiple of 128 (K = %lld)", fn,
                    (long long)K);
  if (R == 0) return KQ_OK;
  if (!scales || !tiled) return kq::fail(KQ_ERR_INVALID_ARG, "%s: NULL pointer", fn);
  const int64_t n_out = (R + 127) / 128 * (K / 128) * 512;
  if (n_out >= ((int64_t)1 << 31) || R * (K / 32) >= ((int64_t)1 << 31))
    return kq::fail(KQ_ERR_UNSUPPORTED, "%s: too large", fn);
  int sms = 0;
  if (int st = kq::sm_count(&sms)) return st;
  int64_t blocks = (n_out + 255) / 256;
  if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
  kq::gemm::sf_tile_kernel<<<(unsigned)blocks, 256, 0, kq::as_stream(stream)>>>(
      scales, (int)R, (int)(K / 32), (int)n_out, tiled);
  return kq::check_launch("sf_tile_kernel launch");
}

int kq_gemm_mxfp4(const uint8_t* a_codes, const uint8_t* a_sf_tiled, const uint8_t* b_codes,
                  const uint8_t* b_sf_tiled, int64_t M, int64_t N, int64_t K, float* Y, void* stream) {
  return kq::gemm_launch(a_codes, a_sf_tiled, b_codes, b_sf_tiled, M, N, K, nullptr, nullptr, Y, false,
                         stream, "kq_gemm_mxfp4");
}

int kq_gemm_mxfp4_rank1(const uint8_t* a_codes, const uint8_t* a_sf_tiled, const uint8_t* b_codes,
                        const uint8_t* b_sf_tiled, int64_t M, int64_t N, int64_t K, const float* mu,
                        const float* wsum, float* Y, void* stream) {
  if (M > 0 && N > 0 && (!mu || !wsum))
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_gemm_mxfp4_rank1: NULL mu or wsum");
  if ((mu && !kq::aligned(mu, 4)) || (wsum && !kq::aligned(wsum, 4)))
    return kq::fail(KQ_ERR_ALIGNMENT, "kq_gemm_mxfp4_rank1: mu and wsum must be 4-byte aligned");
  return kq::gemm_launch(a_codes, a_sf_tiled, b_codes, b_sf_tiled, M, N, K, mu, wsum, Y, false, stream,
                         "kq_gemm_mxfp4_rank1");
}

int kq_gemm_mxfp4_bf16(const uint8_t* a_codes, const uint8_t* a_sf_tiled, const uint8_t* b_codes,
                       const uint8_t* b_sf_tiled, int64_t M, int64_t N, int64_t K, void* Y,
                       void* stream) {
  return kq::gemm_launch(a_codes, a_sf_tiled, b_codes, b_sf_tiled, M, N, K, nullptr, nullptr, Y, true,
                         stream, "kq_gemm_mxfp4_bf16");
}

}  // extern "C"
