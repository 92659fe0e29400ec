// bf16_gemm.cu — C = A B for the layer's projections (bf16 in and out, fp32
// accumulation): A [M][K] and B [K][N] row-major, C [M][N] row-major. The Q/K/V
// projections x W_Q, x W_K, x W_V and the output projection [A_1 ... A_H] W_O of an
// attention layer ("Leave No Context Behind", arXiv 2404.07143, as quoted on
// llm-papers-study.pages.dev, sections 3.1 and 3.6).
//
// Two persistent kernels, 192 threads each: warps 0-3 drain the accumulator (tensor
// memory -> bf16 -> global), warp 4 is the TMA producer, warp 5 allocates tensor
// memory and issues the MMAs from one elected lane; output tiles are taken in the
// order (m, n) with n fastest, so that a block of rows of A is reused from L2 by the
// tiles that need it, and two accumulators let the epilogue of one tile overlap the
// products of the next.
//   gemm_pair_kernel (every N a multiple of 256): 256 x 256 tiles on CTA pairs with
//     cta_group::2 MMAs, epilogue through shared memory and TMA stores; up to three B
//     matrices sharing A in one launch (the layer's Q, K and V projections).
//   gemm_kernel (otherwise): 128 x 128 tiles on one CTA per SM; each k-step brings a
//     128 x 128 tile of A (K-major) and one of B (MN-major) into a 3-stage ring; eight
//     tcgen05 MMAs (K = 16 each) per k-step.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda.h>
#include <cstdint>
#include <cstring>

#include "bf16_path.h"
#include "sm100.cuh"
#include "tma_map.h"

namespace infini {
namespace {

constexpr int kTile = 32768;  // 128 x 128 bf16
constexpr int kSub = 16384;   // one 128 x 64 box
constexpr int kStages = 3;
constexpr int kGemmThreads = 192;
constexpr int kGemmSmem = kStages * 2 * kTile + 256 + 1024;

enum { G_FULL = 0, G_EMPTY = 3, G_AFULL = 6, G_AEMPTY = 8, G_DRAIN = 10, G_COUNT = 11 };

struct GemmParams {
  int tiles_n;     // N / 128 (pair kernel: N / 256, summed over the column groups)
  int ksteps;      // K / 128 (pair kernel: K / 64)
  unsigned tiles;  // (M / 128) * tiles_n (pair kernel: ceil(M / 256) * tiles_n)
  long long ldc;   // N (pair kernel: unused, row strides per group)
};

// The pair kernel's column groups: C_g = A B_g for up to three B matrices that share A
// (the layer's Q, K and V projections of the same x in one launch, so that each
// 128-row block of A is fetched once for all of them). Group g covers the column tiles
// [first[g], first[g + 1]) of the launch.
struct GemmGroups {
  int n;                     // groups (1..3)
  int first[4];              // first column tile of each group, then the total
  __nv_bfloat16* C[3];       // outputs
  long long ldc[3];          // their row strides (elements)
};

__device__ __forceinline__ uint64_t kdesc_g(uint32_t base, int kk) {
  return sdesc(base + (uint32_t)(kk >> 2) * kSub + (uint32_t)(kk & 3) * 32, 16, 1024);
}
__device__ __forceinline__ uint64_t mdesc_g(uint32_t base, int kk) {
  return sdesc(base + (uint32_t)kk * 2048, kSub, 1024);
}

// Tiled 2-D TMA load (box of the map) at element coordinates (c0 = column, c1 = row).
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* m, uint64_t* bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void drain_wait_g(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) break;  // 200 ms
  }
}

__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
            __nv_bfloat16* __restrict__ C, const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * 2 * kTile);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + G_COUNT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int x = 0; x < G_COUNT; ++x)
      mbar_init(&bars[x], (x == G_AEMPTY || x == G_AEMPTY + 1) ? 4u : 1u);
    fence_barrier_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 4) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int it = 0;
      int iss[kStages] = {0, 0, 0};
      for (unsigned t = blockIdx.x; ok && t < p.tiles; t += gridDim.x) {
        const int tm = (int)(t / (unsigned)p.tiles_n), tn = (int)(t % (unsigned)p.tiles_n);
        for (int ks = 0; ks < p.ksteps; ++ks, ++it) {
          const int st = it % kStages;
          const int use = it / kStages;
          if (use > 0 && !mbar_wait(&bars[G_EMPTY + st], (uint32_t)((use - 1) & 1))) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + st * 2 * kTile;
          uint8_t* sb = sa + kTile;
          mbar_arrive_expect_tx(&bars[G_FULL + st], 2 * kTile);
          // A rows [128 tm, +128), columns [128 ks, +128): two 64-column boxes
          tma_load_2d(sa, &tm_a, &bars[G_FULL + st], 128 * ks, 128 * tm);
          tma_load_2d(sa + kSub, &tm_a, &bars[G_FULL + st], 128 * ks + 64, 128 * tm);
          // B rows [128 ks, +128), columns [128 tn, +128)
          tma_load_2d(sb, &tm_b, &bars[G_FULL + st], 128 * tn, 128 * ks);
          tma_load_2d(sb + kSub, &tm_b, &bars[G_FULL + st], 128 * tn + 64, 128 * ks);
          ++iss[st];
        }
      }
      if (!ok)  // let the copies already issued land before the CTA exits
        for (int st = 0; st < kStages; ++st)
          if (iss[st] > 0) drain_wait_g(&bars[G_FULL + st], (uint32_t)((iss[st] - 1) & 1));
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer ----------------
    const uint32_t idesc = idesc_f32acc(1, 0, 1, 128, 128);  // A K-major, B MN-major
    int it = 0, lt = 0;
    for (unsigned t = blockIdx.x; ok && t < p.tiles; t += gridDim.x, ++lt) {
      const int acc = lt & 1, use = lt >> 1;
      if (use > 0 && !mbar_wait_warp(&bars[G_AEMPTY + acc], (uint32_t)((use - 1) & 1))) {
        ok = false;
        break;
      }
      const uint32_t td = tmem + (uint32_t)acc * 128;
      for (int ks = 0; ks < p.ksteps; ++ks, ++it) {
        const int st = it % kStages;
        if (!mbar_wait_warp(&bars[G_FULL + st], (uint32_t)((it / kStages) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint32_t sa = smem_u32(smem + st * 2 * kTile), sb = sa + kTile;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ss(td, kdesc_g(sa, kk), mdesc_g(sb, kk), idesc, (ks > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&bars[G_EMPTY + st]);  // the stage may be refilled
          if (ks == p.ksteps - 1) mma_commit(&bars[G_AFULL + acc]);
        }
        __syncwarp();
      }
    }
    // no MMA may still run when the CTA frees tensor memory
    if (elect_one()) mma_commit(&bars[G_DRAIN]);
    __syncwarp();
    drain_wait_g(&bars[G_DRAIN], 0);
  } else {
    // ---------------- epilogue (warps 0-3): row r of each output tile ----------------
    const int r = warp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    int lt = 0;
    for (unsigned t = blockIdx.x; ok && t < p.tiles; t += gridDim.x, ++lt) {
      const int acc = lt & 1;
      if (!mbar_wait_warp(&bars[G_AFULL + acc], (uint32_t)((lt >> 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int tm = (int)(t / (unsigned)p.tiles_n), tn = (int)(t % (unsigned)p.tiles_n);
      uint32_t v[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(tmem + (uint32_t)acc * 128 + lane_off + 32 * c,
                  *reinterpret_cast<uint32_t(*)[32]>(v + 32 * c));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive_warp(&bars[G_AEMPTY + acc]);  // the accumulator may take the next tile
      __nv_bfloat16* dst = C + (size_t)(128 * tm + r) * p.ldc + 128 * tn;
#pragma unroll
      for (int u = 0; u < 16; ++u)
        *reinterpret_cast<uint4*>(dst + 8 * u) = make_uint4(
            pack_bf16x2(__uint_as_float(v[8 * u]), __uint_as_float(v[8 * u + 1])),
            pack_bf16x2(__uint_as_float(v[8 * u + 2]), __uint_as_float(v[8 * u + 3])),
            pack_bf16x2(__uint_as_float(v[8 * u + 4]), __uint_as_float(v[8 * u + 5])),
            pack_bf16x2(__uint_as_float(v[8 * u + 6]), __uint_as_float(v[8 * u + 7])));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// The same GEMM with 256 x 256 output tiles (N a multiple of 256) on a CTA pair (a
// cluster of two CTAs, one per SM, driving tcgen05 MMAs with cta_group::2). Each k-step
// of 64 brings into each CTA its 128 rows of A (one 16 KB box, K-major) and its 128
// columns of B (two 8 KB boxes of 64 columns, MN-major), into a 6-stage ring; both
// CTAs' copies complete on the even CTA's barrier, and the even CTA issues four pair
// MMAs (M = 256, N = 256, K = 16) per k-step into one of two 256-column accumulators,
// each CTA's tensor memory holding its own 128 rows of the tile. Per FLOP an SM
// streams two thirds of what a 128 x 256 tile on one SM needs through L2, and the ring
// covers more of the latency. In both CTAs four epilogue warps drain their own rows of
// the accumulator 64 columns at a time (tensor memory -> bf16 -> a swizzled staging
// buffer -> a TMA store of 32 rows x 64 columns, full 128-byte lines), and release the
// accumulator on the even CTA's barrier once it has been read.
constexpr int kPStages = 5;
constexpr int kPA = 16384, kPB = 16384, kPStage = kPA + kPB;
// epilogue staging: per epilogue warp two 4 KB buffers (32 rows x 64 columns, 128-byte
// swizzle), written from registers and sent to C by TMA stores
constexpr int kPOut = 4 * 2 * 4096;
constexpr int kGemmPSmem = kPStages * kPStage + kPOut + 256 + 1024;
// FULL (the even CTA's: 1 arrival with the pair's bytes), EMPTY, AFULL (arrivals
// sent to both CTAs by the MMA commits), AEMPTY (the even CTA's: 4 warps of each
// CTA), DRAIN (both CTAs: every MMA issued has completed)
enum {
  P_FULL = 0,
  P_EMPTY = P_FULL + kPStages,
  P_AFULL = P_EMPTY + kPStages,
  P_AEMPTY = P_AFULL + 2,
  P_DRAIN = P_AEMPTY + 2,
  P_COUNT = P_DRAIN + 1
};
static_assert(P_COUNT * 8 + 4 <= 256, "barrier area");

__device__ __forceinline__ int gemm_group(const GemmGroups& gr, int tn) {
  return tn < gr.first[1] ? 0 : (tn < gr.first[2] ? 1 : 2);
}

// TMA load into this CTA's shared memory whose completion is counted on an mbarrier of
// either CTA of the pair (cluster-window address).
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* m,
                                                 uint32_t bar_cluster, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}

// First row of this CTA's half of row tile tm. A half that lies wholly past the last
// row (M an odd number of 128-row blocks) loads the last 128 rows instead: its products
// are never stored, and every copy stays inside the matrix.
__device__ __forceinline__ int a_row(int tm, uint32_t rank, long long M) {
  const long long r = 256ll * tm + 128 * (long long)rank;
  return (int)(r < M ? r : M - 128);
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, const void* smem_src, int c0,
                                             int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(m)),
      "r"(smem_u32(smem_src)), "r"(c0), "r"(c1)
      : "memory");
}

// Until at most one of this thread's bulk store groups is still reading shared memory.
__device__ __forceinline__ void bulk_wait_group_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

struct PairOut {
  CUtensorMap c[3];  // C_g, box 64 columns x 32 rows, 128-byte swizzle
};

__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b0,
                 const __grid_constant__ CUtensorMap tm_b1, const __grid_constant__ CUtensorMap tm_b2,
                 const __grid_constant__ PairOut out, const GemmParams p, const GemmGroups gr,
                 const long long M) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stage_out = smem + kPStages * kPStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(stage_out + kPOut);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + P_COUNT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool lead = rank == 0;
  const unsigned pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  if (threadIdx.x == 0) {
    for (int x = 0; x < P_COUNT; ++x)
      mbar_init(&bars[x], (x == P_AEMPTY || x == P_AEMPTY + 1) ? 8u : 1u);
    fence_barrier_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b0);
    if (gr.n > 1) tma_prefetch_desc(&tm_b1);
    if (gr.n > 2) tma_prefetch_desc(&tm_b2);
  }
  if (warp == 5) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers initialised in both CTAs before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 4) {
    if (lane == 0) {
      int it = 0;
      int iss[kPStages] = {};
      for (unsigned t = pair; ok && t < p.tiles; t += npairs) {
        const int tm = (int)(t / (unsigned)p.tiles_n), tn = (int)(t % (unsigned)p.tiles_n);
        const int g = gemm_group(gr, tn), tl = tn - gr.first[g];
        const CUtensorMap* tmb = g == 0 ? &tm_b0 : (g == 1 ? &tm_b1 : &tm_b2);
        for (int ks = 0; ks < p.ksteps; ++ks, ++it) {
          const int st = it % kPStages, use = it / kPStages;
          if (use > 0 && !mbar_wait(&bars[P_EMPTY + st], (uint32_t)((use - 1) & 1))) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + st * kPStage;
          uint8_t* sb = sa + kPA;
          if (lead) mbar_arrive_expect_tx(&bars[P_FULL + st], 2 * kPStage);
          const uint32_t full = smem_cluster_addr(&bars[P_FULL + st], 0);
          tma_load_2d_pair(sa, &tm_a, full, 64 * ks, a_row(tm, rank, M));
#pragma unroll
          for (int a2 = 0; a2 < 2; ++a2)
            tma_load_2d_pair(sb + a2 * 8192, tmb, full, 256 * tl + 128 * (int)rank + 64 * a2,
                             64 * ks);
          ++iss[st];
        }
      }
      // every copy into this CTA's ring has landed (and every arrival on its EMPTY
      // barriers) once the last use of each stage has been released
      for (int st = 0; st < kPStages; ++st)
        if (iss[st] > 0) drain_wait_g(&bars[P_EMPTY + st], (uint32_t)((iss[st] - 1) & 1));
    }
    __syncwarp();
  } else if (warp == 5) {
    if (lead) {
      const uint32_t idesc = idesc_f32acc(1, 0, 1, 256, 256);
      int it = 0, lt = 0;
      for (unsigned t = pair; ok && t < p.tiles; t += npairs, ++lt) {
        const int acc = lt & 1, use = lt >> 1;
        if (use > 0 && !mbar_wait_warp(&bars[P_AEMPTY + acc], (uint32_t)((use - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t td = tmem + (uint32_t)acc * 256;
        for (int ks = 0; ks < p.ksteps; ++ks, ++it) {
          const int st = it % kPStages;
          if (!mbar_wait_warp(&bars[P_FULL + st], (uint32_t)((it / kPStages) & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
            const uint32_t sa = smem_u32(smem + st * kPStage), sb = sa + kPA;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16_ss_pair(td, sdesc(sa + (uint32_t)kk * 32, 16, 1024),
                               sdesc(sb + (uint32_t)kk * 2048, 8192, 1024), idesc,
                               (ks > 0 || kk > 0) ? 1u : 0u);
            mma_commit_pair(&bars[P_EMPTY + st], 3);
            if (ks == p.ksteps - 1) mma_commit_pair(&bars[P_AFULL + acc], 3);
          }
          __syncwarp();
        }
      }
      if (elect_one()) mma_commit_pair(&bars[P_DRAIN], 3);
      __syncwarp();
      // both CTAs' epilogues have released every accumulator use (their arrivals on
      // this CTA's barriers have landed)
      if (lane == 0)
        for (int acc = 0; acc < 2; ++acc) {
          const int uses = (lt + 1 - acc) / 2;
          if (uses > 0) drain_wait_g(&bars[P_AEMPTY + acc], (uint32_t)((uses - 1) & 1));
        }
      __syncwarp();
    }
    // no MMA into either CTA's tensor memory is in flight past this point
    if (lane == 0) drain_wait_g(&bars[P_DRAIN], 0);
    __syncwarp();
  } else {
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    uint8_t* sbuf = stage_out + warp * 8192;
    int lt = 0, chunk = 0;
    for (unsigned t = pair; ok && t < p.tiles; t += npairs, ++lt) {
      const int acc = lt & 1;
      if (!mbar_wait_warp(&bars[P_AFULL + acc], (uint32_t)((lt >> 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int tm = (int)(t / (unsigned)p.tiles_n), tn = (int)(t % (unsigned)p.tiles_n);
      const int g = gemm_group(gr, tn);
      const long long row0 = 256ll * tm + 128 * (int)rank + 32 * warp;  // this warp's rows
      const int col0 = 256 * (tn - gr.first[g]);
#pragma unroll 1
      for (int c4 = 0; c4 < 4; ++c4, ++chunk) {
        uint8_t* buf = sbuf + (chunk & 1) * 4096;
        uint32_t v[64];
        tmem_ld32(tmem + (uint32_t)acc * 256 + lane_off + 64 * c4,
                  *reinterpret_cast<uint32_t(*)[32]>(v));
        tmem_ld32(tmem + (uint32_t)acc * 256 + lane_off + 64 * c4 + 32,
                  *reinterpret_cast<uint32_t(*)[32]>(v + 32));
        tmem_wait_ld();
        if (c4 == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(smem_cluster_addr(&bars[P_AEMPTY + acc], 0));
        }
        // the store that last read this buffer (two chunks back) has finished reading
        if (lane == 0 && chunk >= 2) bulk_wait_group_read1();
        __syncwarp();
        const uint32_t rowb = smem_u32(buf) + (uint32_t)lane * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          st_shared_v4(rowb + (uint32_t)((u ^ (lane & 7)) * 16),
                        pack_bf16x2(__uint_as_float(v[8 * u]), __uint_as_float(v[8 * u + 1])),
                        pack_bf16x2(__uint_as_float(v[8 * u + 2]), __uint_as_float(v[8 * u + 3])),
                        pack_bf16x2(__uint_as_float(v[8 * u + 4]), __uint_as_float(v[8 * u + 5])),
                        pack_bf16x2(__uint_as_float(v[8 * u + 6]), __uint_as_float(v[8 * u + 7])));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          // rows past the end of C are clipped by the store; a block wholly past it is
          // not sent
          if (row0 < M) tma_store_2d(&out.c[g], buf, col0 + 64 * c4, (int)row0);
          tma_store_commit();
        }
      }
    }
    if (lane == 0) tma_store_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync_all();  // both CTAs done with tensor memory and with each other's barriers
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// 2-D bf16 map over a row-major [rows][cols] matrix: box 64 columns x 128 rows,
// 128-byte swizzle (one box row is one 128-byte swizzle row).
bool make_bf16_map2(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows = 128) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t bf16_gemm_set_attributes() {
  const cudaError_t e =
      cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kGemmPSmem);
}

namespace {
// CTAs of the pair kernel that can be resident at once (two per co-resident cluster),
// looked up once per device.
int pair_kernel_ctas() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cached[dev] > 0) return cached[dev];
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((unsigned)(sms & ~1));
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = kGemmPSmem;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, gemm_pair_kernel, &cfg) != cudaSuccess ||
      clusters < 1) {
    cudaGetLastError();
    return 0;
  }
  cached[dev] = 2 * clusters;
  return cached[dev];
}
}  // namespace

cudaError_t bf16_gemm_grouped_launch(const __nv_bfloat16* A, const __nv_bfloat16* const* B,
                                     __nv_bfloat16* const* C, const int* N, int ngroups,
                                     long long M, int K, cudaStream_t stream) {
  if (ngroups < 1 || ngroups > 3 || M <= 0 || K <= 0 || M % 128 || K % 128 || M >= (1ll << 31))
    return cudaErrorInvalidValue;
  const int ctas = pair_kernel_ctas();
  if (ctas < 2) return cudaErrorLaunchOutOfResources;
  CUtensorMap ma, mb[3];
  PairOut out;
  if (!make_bf16_map2(&ma, A, (uint64_t)M, (uint64_t)K, 128)) return cudaErrorInvalidValue;
  GemmGroups gr;
  memset(&gr, 0, sizeof(gr));
  gr.n = ngroups;
  for (int g = 0; g < ngroups; ++g) {
    if (N[g] <= 0 || N[g] % 256 != 0) return cudaErrorInvalidValue;
    if (!make_bf16_map2(&mb[g], B[g], (uint64_t)K, (uint64_t)N[g], 64)) return cudaErrorInvalidValue;
    if (!make_bf16_map2(&out.c[g], C[g], (uint64_t)M, (uint64_t)N[g], 32))
      return cudaErrorInvalidValue;
    gr.C[g] = C[g];
    gr.ldc[g] = N[g];
    gr.first[g + 1] = gr.first[g] + N[g] / 256;
  }
  for (int g = ngroups; g < 3; ++g) {
    mb[g] = mb[0];
    out.c[g] = out.c[0];
    gr.first[g + 1] = gr.first[g];
    gr.C[g] = C[0];
    gr.ldc[g] = 0;
  }
  GemmParams p;
  p.tiles_n = gr.first[ngroups];
  p.ksteps = K / 64;
  const long long tiles = ((M + 255) / 256) * (long long)p.tiles_n;
  if (tiles >= (1ll << 31)) return cudaErrorInvalidValue;
  p.tiles = (unsigned)tiles;
  p.ldc = 0;
  const unsigned pairs = p.tiles < (unsigned)(ctas / 2) ? p.tiles : (unsigned)(ctas / 2);
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = kGemmPSmem;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_pair_kernel, ma, mb[0], mb[1], mb[2], out, p, gr, M);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t bf16_gemm_launch(const __nv_bfloat16* A, const __nv_bfloat16* B, __nv_bfloat16* C,
                             long long M, int N, int K, cudaStream_t stream) {
  if (M <= 0 || N <= 0 || K <= 0 || M % 128 || N % 128 || K % 128) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (N % 256 == 0) {  // 128 x 256 tiles
    const __nv_bfloat16* Bs[1] = {B};
    __nv_bfloat16* Cs[1] = {C};
    const int Ns[1] = {N};
    return bf16_gemm_grouped_launch(A, Bs, Cs, Ns, 1, M, K, stream);
  }
  CUtensorMap ma, mb;
  if (!make_bf16_map2(&ma, A, (uint64_t)M, (uint64_t)K) ||
      !make_bf16_map2(&mb, B, (uint64_t)K, (uint64_t)N))
    return cudaErrorInvalidValue;
  GemmParams p;
  p.tiles_n = N / 128;
  p.ksteps = K / 128;
  const long long tiles = (M / 128) * (long long)(N / 128);
  if (tiles >= (1ll << 31)) return cudaErrorInvalidValue;
  p.tiles = (unsigned)tiles;
  p.ldc = N;
  const unsigned grid = p.tiles < (unsigned)sms ? p.tiles : (unsigned)sms;
  gemm_kernel<<<grid, kGemmThreads, kGemmSmem, stream>>>(ma, mb, C, p);
  return cudaGetLastError();
}

}  // namespace infini
