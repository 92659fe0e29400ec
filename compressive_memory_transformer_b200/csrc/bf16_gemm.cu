// bf16_gemm.cu — C = A B for the layer's projections (bf16 in and out, fp32
// accumulation): A [M][K] and B [K][N] row-major, C [M][N] row-major. The Q/K/V
// projections x W_Q, x W_K, x W_V and the output projection [A_1 ... A_H] W_O of an
// attention layer ("Leave No Context Behind", arXiv 2404.07143, as quoted on
// llm-papers-study.pages.dev, sections 3.1 and 3.6).
//
// Persistent kernel, one CTA per SM, 192 threads: warps 0-3 drain the accumulator
// (tensor memory -> bf16 -> global), warp 4 is the TMA producer, warp 5 allocates
// tensor memory and issues the MMAs from one elected lane. Output tiles are 128 x 128,
// taken in the order (m, n) with n fastest so that a 128-row block of A is reused
// from L2 by the N/128 tiles that need it. Each k-step brings a 128 x 128 tile of A
// (K-major) and one of B (MN-major) into a 3-stage ring; eight tcgen05 MMAs
// (K = 16 each) accumulate into one of two 128-column accumulators, so the epilogue
// of one tile overlaps the products of the next.
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
  int tiles_n;     // N / 128 (wide kernel: N / 256, summed over the column groups)
  int ksteps;      // K / 128 (wide kernel: K / 64)
  unsigned tiles;  // (M / 128) * tiles_n
  long long ldc;   // N
};

// The wide kernel's column groups: C_g = A B_g for up to three B matrices that share A
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

// The same GEMM with 128 x 256 output tiles (N a multiple of 256): each k-step of 64
// brings A [128 m][64 k] (one 16 KB box, K-major) and B [64 k][256 n] (four 8 KB
// boxes of 64 columns, MN-major) into a 4-stage ring; four MMAs (N = 256, K = 16)
// per k-step into one of two 256-column accumulators. Per FLOP it streams a quarter
// less through L2 than the 128 x 128 tiles.
constexpr int kWStages = 4;
constexpr int kWA = 16384, kWB = 32768, kWStage = kWA + kWB;
constexpr int kGemmWSmem = kWStages * kWStage + 256 + 1024;

__device__ __forceinline__ int gemm_group(const GemmGroups& gr, int tn) {
  return tn < gr.first[1] ? 0 : (tn < gr.first[2] ? 1 : 2);
}

__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_wide_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b0,
                 const __grid_constant__ CUtensorMap tm_b1, const __grid_constant__ CUtensorMap tm_b2,
                 const GemmParams p, const GemmGroups gr) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWStages * kWStage);
  // FULL [0, 4), EMPTY [4, 8), AFULL 8-9, AEMPTY 10-11 (4 warp arrivals), DRAIN 12
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int x = 0; x < 13; ++x) mbar_init(&bars[x], (x == 10 || x == 11) ? 4u : 1u);
    fence_barrier_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b0);
    if (gr.n > 1) tma_prefetch_desc(&tm_b1);
    if (gr.n > 2) tma_prefetch_desc(&tm_b2);
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 4) {
    if (lane == 0) {
      int it = 0;
      int iss[kWStages] = {0, 0, 0, 0};
      for (unsigned t = blockIdx.x; ok && t < p.tiles; t += gridDim.x) {
        const int tm = (int)(t / (unsigned)p.tiles_n), tn = (int)(t % (unsigned)p.tiles_n);
        const int g = gemm_group(gr, tn), tl = tn - gr.first[g];
        const CUtensorMap* tmb = g == 0 ? &tm_b0 : (g == 1 ? &tm_b1 : &tm_b2);
        for (int ks = 0; ks < p.ksteps; ++ks, ++it) {
          const int st = it % kWStages, use = it / kWStages;
          if (use > 0 && !mbar_wait(&bars[4 + st], (uint32_t)((use - 1) & 1))) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + st * kWStage;
          uint8_t* sb = sa + kWA;
          mbar_arrive_expect_tx(&bars[st], kWStage);
          tma_load_2d(sa, &tm_a, &bars[st], 64 * ks, 128 * tm);
#pragma unroll
          for (int a4 = 0; a4 < 4; ++a4)
            tma_load_2d(sb + a4 * 8192, tmb, &bars[st], 256 * tl + 64 * a4, 64 * ks);
          ++iss[st];
        }
      }
      if (!ok)
        for (int st = 0; st < kWStages; ++st)
          if (iss[st] > 0) drain_wait_g(&bars[st], (uint32_t)((iss[st] - 1) & 1));
    }
  } else if (warp == 5) {
    const uint32_t idesc = idesc_f32acc(1, 0, 1, 128, 256);
    int it = 0, lt = 0;
    for (unsigned t = blockIdx.x; ok && t < p.tiles; t += gridDim.x, ++lt) {
      const int acc = lt & 1, use = lt >> 1;
      if (use > 0 && !mbar_wait_warp(&bars[10 + acc], (uint32_t)((use - 1) & 1))) {
        ok = false;
        break;
      }
      const uint32_t td = tmem + (uint32_t)acc * 256;
      for (int ks = 0; ks < p.ksteps; ++ks, ++it) {
        const int st = it % kWStages;
        if (!mbar_wait_warp(&bars[st], (uint32_t)((it / kWStages) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint32_t sa = smem_u32(smem + st * kWStage), sb = sa + kWA;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(td, sdesc(sa + (uint32_t)kk * 32, 16, 1024),
                        sdesc(sb + (uint32_t)kk * 2048, 8192, 1024), idesc,
                        (ks > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&bars[4 + st]);
          if (ks == p.ksteps - 1) mma_commit(&bars[8 + acc]);
        }
        __syncwarp();
      }
    }
    if (elect_one()) mma_commit(&bars[12]);
    __syncwarp();
    drain_wait_g(&bars[12], 0);
  } else {
    const int r = warp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    int lt = 0;
    for (unsigned t = blockIdx.x; ok && t < p.tiles; t += gridDim.x, ++lt) {
      const int acc = lt & 1;
      if (!mbar_wait_warp(&bars[8 + acc], (uint32_t)((lt >> 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int tm = (int)(t / (unsigned)p.tiles_n), tn = (int)(t % (unsigned)p.tiles_n);
      const int g = gemm_group(gr, tn);
      __nv_bfloat16* dst = gr.C[g] + (size_t)(128 * tm + r) * gr.ldc[g] + 256 * (tn - gr.first[g]);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t v[128];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld32(tmem + (uint32_t)acc * 256 + lane_off + 128 * hf + 32 * c,
                    *reinterpret_cast<uint32_t(*)[32]>(v + 32 * c));
        tmem_wait_ld();
        if (hf == 1) {
          tc_fence_before();
          mbar_arrive_warp(&bars[10 + acc]);  // the accumulator may take the next tile
        }
#pragma unroll
        for (int u = 0; u < 16; ++u)
          *reinterpret_cast<uint4*>(dst + 128 * hf + 8 * u) = make_uint4(
              pack_bf16x2(__uint_as_float(v[8 * u]), __uint_as_float(v[8 * u + 1])),
              pack_bf16x2(__uint_as_float(v[8 * u + 2]), __uint_as_float(v[8 * u + 3])),
              pack_bf16x2(__uint_as_float(v[8 * u + 4]), __uint_as_float(v[8 * u + 5])),
              pack_bf16x2(__uint_as_float(v[8 * u + 6]), __uint_as_float(v[8 * u + 7])));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
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
  return cudaFuncSetAttribute(gemm_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kGemmWSmem);
}

cudaError_t bf16_gemm_grouped_launch(const __nv_bfloat16* A, const __nv_bfloat16* const* B,
                                     __nv_bfloat16* const* C, const int* N, int ngroups,
                                     long long M, int K, cudaStream_t stream) {
  if (ngroups < 1 || ngroups > 3 || M <= 0 || K <= 0 || M % 128 || K % 128)
    return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  CUtensorMap ma, mb[3];
  if (!make_bf16_map2(&ma, A, (uint64_t)M, (uint64_t)K, 128)) return cudaErrorInvalidValue;
  GemmGroups gr;
  memset(&gr, 0, sizeof(gr));
  gr.n = ngroups;
  for (int g = 0; g < ngroups; ++g) {
    if (N[g] <= 0 || N[g] % 256 != 0) return cudaErrorInvalidValue;
    if (!make_bf16_map2(&mb[g], B[g], (uint64_t)K, (uint64_t)N[g], 64)) return cudaErrorInvalidValue;
    gr.C[g] = C[g];
    gr.ldc[g] = N[g];
    gr.first[g + 1] = gr.first[g] + N[g] / 256;
  }
  for (int g = ngroups; g < 3; ++g) {
    mb[g] = mb[0];
    gr.first[g + 1] = gr.first[g];
    gr.C[g] = C[0];
    gr.ldc[g] = 0;
  }
  GemmParams p;
  p.tiles_n = gr.first[ngroups];
  p.ksteps = K / 64;
  const long long tiles = (M / 128) * (long long)p.tiles_n;
  if (tiles >= (1ll << 31)) return cudaErrorInvalidValue;
  p.tiles = (unsigned)tiles;
  p.ldc = 0;
  const unsigned grid = p.tiles < (unsigned)sms ? p.tiles : (unsigned)sms;
  gemm_wide_kernel<<<grid, kGemmThreads, kGemmWSmem, stream>>>(ma, mb[0], mb[1], mb[2], p, gr);
  return cudaGetLastError();
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
