// bf16_bwd.cu — gradient of the bf16 forward (d = 128, [B, H, L, d], N a multiple of
// 128 and L a multiple of N).
//
// The layer ("Leave No Context Behind", arXiv 2404.07143, as quoted on
// llm-papers-study.pages.dev, sections 3.1, 3.3-3.5) is, per head and segment s,
//   out = g A_mem + (1 - g) A_dot,   A_dot = softmax(Q K^T / sqrt(d) + mask) V,
//   A_mem = sigma(Q) M_{s-1} / (sigma(Q) z_{s-1}),
//   M_s = M_{s-1} + sigma(K)^T V                 (Linear)
//   M_s = M_{s-1} + sigma(K)^T (V - R),  R = sigma(K) M_{s-1} / (sigma(K) z_{s-1})  (Delta)
//   z_s = z_{s-1} + sum_t sigma(K_t).
// Its gradient is the chain rule through those steps in reverse segment order. With
// dM_s, dz_s the gradients of the state after segment s:
//   retrieval: dnum = g dout / den, dden = -rowsum(g dout * A_mem) / den,
//              dsigma(Q) = dnum M^T + dden z^T, and (M_{s-1}, z_{s-1}) receive
//              GM_s = sigma(Q)^T dnum and Gz_s = sigma(Q)^T dden;
//   Linear:    dM_{s-1} = dM_s + GM_s;  dsigma(K) = V dM_s^T + dz_s;  dV += sigma(K) dM_s;
//   Delta:     dU = sigma(K) dM_s (U = V - R), dV += dU, and through R
//              dM_{s-1} = dM_s - G_s dM_s + GM_s with G_s = sigma(K)^T diag(1/den_K) sigma(K)
//              (the same symmetric matrix the forward's state kernel builds),
//              dsigma(K) = U dM_s^T - (dU / den_K) M^T + ddenR z^T + dz_s,
//              ddenR = rowsum(dU * R) / den_K, dz_{s-1} = dz_s + sigma(K)^T ddenR + Gz_s;
//   attention: the usual softmax backward of the local causal attention, scaled by
//              (1 - g); dbeta = g (1 - g) sum dout * (A_mem - A_dot).
// Rows whose denominator is exactly 0 retrieve the constant 0 and pass no gradient.
//
// Kernels, in launch order (after the forward's state path has rebuilt M_{s-1} as
// bf16 hi/lo, z_{s-1} and, for Delta, every segment's G_s):
//   dq     (head, segment, query tile): two sweeps over the key tiles; the first
//          gives each row's log-sum-exp and D' = dout . A_dot, the second
//          dQ = sum_j dS_j K_j; then the retrieval's backward of its query rows
//          (dsigma(Q), and the tile's partials of GM_s and Gz_s); writes dq, the row
//          statistics and the tile's sums for dbeta.
//   chain  (head, 32-column block): dM_s for s = S-1 .. 0 (bf16 hi/lo stack), dM_in.
//   dz     (head, Linear): dz_s for every segment, dz_in.
//   dkdv   (head, segment, key tile): over the query tiles at or after it,
//          dV = sum_i (1-g) P_i^T dout_i and dK = sum_i dS_i^T Q_i from S^T = K Q^T
//          and dP'^T = V dout^T; then the memory update's backward of its key rows
//          (dV += sigma(K) dM_s, dsigma(K), and for Delta sigma(K)^T ddenR per tile);
//          writes dk, dv.
//   dz, dk_dz (Delta): dz_s for every segment (it needs every tile's sigma(K)^T
//          ddenR), dz_in, then dk += dz_s * sigma'(K).
//   dbeta  : per head, summed over batch rows, segments and tiles in a fixed order.
// Every product is a bf16 tcgen05 MMA (fp32 accumulation in tensor memory) on
// 128B-swizzled shared-memory tiles, in the operand forms the forward uses: A, B
// both K-major (Q K^T), A in tensor memory with B MN-major (P V), and A, B both
// MN-major (sigma(K)^T V); the Delta chain uses the forward chain's tf32 form.
// Thread r of a 128-thread warpgroup owns tile row r (tensor-memory lane r).
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

constexpr int D = 128;
constexpr int kTile = 32768;  // 128 x 128 bf16
constexpr int kSub = 16384;   // one 128 x 64 box (128-byte rows)

// ---------------------------------------------------------------------------
// tiles, descriptors, products
// ---------------------------------------------------------------------------
// Byte offset of 16-byte unit u (0..15: features 8u .. 8u+7) of row r of a tile
// stored as two 64-column boxes with the 128-byte swizzle (the TMA layout).
__device__ __forceinline__ uint32_t toff(int r, int u) {
  return (uint32_t)(u >> 3) * kSub + sw128((uint32_t)r, (uint32_t)(u & 7));
}
__device__ __forceinline__ uint4 ld_unit(const uint8_t* t, int r, int u) {
  return *reinterpret_cast<const uint4*>(t + toff(r, u));
}
__device__ __forceinline__ void st_unit(uint8_t* t, int r, int u, const float (&f)[8]) {
  *reinterpret_cast<uint4*>(t + toff(r, u)) =
      make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                 pack_bf16x2(f[6], f[7]));
}
__device__ __forceinline__ void unpack8(const uint4& raw, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 t = __bfloat1622float2(h[e]);
    f[2 * e] = t.x;
    f[2 * e + 1] = t.y;
  }
}
// element (r, c) of a tile
__device__ __forceinline__ float ld_elem(const uint8_t* t, int r, int c) {
  const __nv_bfloat16* p = reinterpret_cast<const __nv_bfloat16*>(t + toff(r, c >> 3)) + (c & 7);
  return __bfloat162float(*p);
}

// sigma = ELU + 1 and its derivative (1 for x > 0, e^x otherwise), full-precision exp
__device__ __forceinline__ float sig(float x) { return x > 0.f ? x + 1.f : expf(x); }
__device__ __forceinline__ float dsig(float x) { return x > 0.f ? 1.f : expf(x); }

__device__ __forceinline__ uint64_t kdesc(uint32_t base, int kk) {
  return sdesc(base + (uint32_t)(kk >> 2) * kSub + (uint32_t)(kk & 3) * 32, 16, 1024);
}
__device__ __forceinline__ uint64_t mdesc(uint32_t base, int kk) {
  return sdesc(base + (uint32_t)kk * 2048, kSub, 1024);
}
constexpr uint32_t kIdKK = idesc_f32acc(1, 0, 0, 128, 128);
constexpr uint32_t kIdKM = idesc_f32acc(1, 0, 1, 128, 128);

// D (+)= A B^T: A[m][k] and B[n][k] are tiles (rows m and n, 128 k each)
__device__ __forceinline__ void gemm_kk(uint32_t d, const uint8_t* a, const uint8_t* b, bool acc) {
  const uint32_t sa = smem_u32(a), sb = smem_u32(b);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    mma_bf16_ss(d, kdesc(sa, kk), kdesc(sb, kk), kIdKK, (acc || kk > 0) ? 1u : 0u);
}
// D (+)= A X: A[m][k] and X[k][n] are tiles
__device__ __forceinline__ void gemm_km(uint32_t d, const uint8_t* a, const uint8_t* x, bool acc) {
  const uint32_t sa = smem_u32(a), sx = smem_u32(x);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    mma_bf16_ss(d, kdesc(sa, kk), mdesc(sx, kk), kIdKM, (acc || kk > 0) ? 1u : 0u);
}
// Both boxes of a 128-row tile of a [B, H, L, 128] tensor.
__device__ __forceinline__ void load_rows(uint8_t* dst, const CUtensorMap* m, uint64_t* bar, int row,
                                          int h, int b) {
  tma_load_4d(dst, m, bar, 0, row, h, b);
  tma_load_4d(dst + kSub, m, bar, 64, row, h, b);
}
// Both boxes of a [128][128] plane of a 3-D map.
__device__ __forceinline__ void load_plane(uint8_t* dst, const CUtensorMap* m, uint64_t* bar,
                                           int plane) {
  tma_load_3d(dst, m, bar, 0, 0, plane);
  tma_load_3d(dst + kSub, m, bar, 64, 0, plane);
}

// Bounded wait used only while draining after an error.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) break;  // 200 ms
  }
}

struct BwdParams {
  long long L;       // tokens per (batch row, head)
  int N, S, T, H;    // T = N / 128 tiles per segment
  unsigned tiles;    // BH * S * T
  FastDiv divT, divS;
  float sl;          // log2(e) / sqrt(d)
  float rsd;         // 1 / sqrt(d)
};

// grid index -> (bh, s, tile)
__device__ __forceinline__ void decode3(const BwdParams& p, unsigned u, int& bh, int& s, int& t) {
  const unsigned seg = p.divT.div(u);
  t = (int)(u - seg * (unsigned)p.T);
  const unsigned b = p.divS.div(seg);
  s = (int)(seg - b * (unsigned)p.S);
  bh = (int)b;
}

// ---------------------------------------------------------------------------
// chain: grid = (BH, 4), block 160. Column block cb covers dM[:, 32cb .. 32cb+31];
// threads 0..127 own one row (32 fp32 values); warp 4 issues the copies of G and the
// tf32 products (Delta). For s = S-1 .. 0: write X = dM_s as bf16 hi/lo into the
// stack, then X += GM_s (Linear) or X += GM_s - G_s X (Delta), GM_s being the sum of
// the segment's per-query-tile partials; finally dM_in = X.
// ---------------------------------------------------------------------------
constexpr int kChainThreads = 160;
constexpr int kGBytes = D * D * 4;    // 64 KB
constexpr int kXtBytes = 32 * D * 4;  // 16 KB: the X block transposed [32][128], tf32
constexpr int kChainSmem = 2 * kGBytes + kXtBytes + 1024 + 256;

__device__ __forceinline__ uint32_t tf32_rna(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

__global__ void __launch_bounds__(kChainThreads, 1)
chain_bwd_kernel(const __grid_constant__ CUtensorMap tm_g, const float* __restrict__ GMp,
                 const float* dM_out, float* dM_in, __nv_bfloat16* __restrict__ dMs, int S,
                 int CH, int T, int mode) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sG = smem;
  uint8_t* sXt = smem + 2 * kGBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * kGBytes + kXtBytes);
  uint64_t* bar_g = bars;        // [2] G chunk landed
  uint64_t* bar_xt = bars + 2;   // X^T written (4 warp arrivals)
  uint64_t* bar_mma = bars + 3;  // one G_c X product done
  uint64_t* bar_seg = bars + 4;  // G_s X of a whole segment done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 5);

  const int bh = blockIdx.x, cb = blockIdx.y, tid = threadIdx.x, warp = tid >> 5;
  const int c0 = 32 * cb;
  const bool delta = mode == 1;
  if (tid == 0) {
    mbar_init(&bar_g[0], 1);
    mbar_init(&bar_g[1], 1);
    mbar_init(bar_xt, 4);
    mbar_init(bar_mma, 1);
    mbar_init(bar_seg, 1);
    fence_barrier_init();
  }
  if (warp == 4) {
    tmem_alloc(tmem_slot, 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  bool ok = true;

  if (warp == 4) {
    if (delta) {
      // load n of the sequence (s = S-1-n/CH, chunk n%CH): G plane of dpart
      int g_iss[2] = {0, 0}, g_cons[2] = {0, 0};
      auto load_g = [&](int n, int buf) {
        if (elect_one()) {
          const int s = S - 1 - n / CH, c = n % CH;
          mbar_arrive_expect_tx(&bar_g[buf], kGBytes);
          const int plane = ((bh * S + s) * CH + c) * 2 + 1;
#pragma unroll
          for (int bx = 0; bx < 4; ++bx)
            tma_load_3d(sG + buf * kGBytes + bx * (D * 128), &tm_g, &bar_g[buf], bx * 32, 0,
                        plane);
        }
        __syncwarp();
        ++g_iss[buf];
      };
      const uint32_t idesc = idesc_f32acc(2, 0, 0, 128, 32);
      const int total = S * CH;
      int n = 0;
      load_g(0, 0);
      for (int q = 0; q < S && ok; ++q) {
        if (!mbar_wait_warp(bar_xt, (uint32_t)(q & 1))) {
          ok = false;
          break;
        }
        for (int c = 0; c < CH; ++c, ++n) {
          const int buf = n & 1;
          if (n + 1 < total) load_g(n + 1, buf ^ 1);
          if (!mbar_wait_warp(&bar_g[buf], (uint32_t)((n >> 1) & 1))) {
            ok = false;
            break;
          }
          ++g_cons[buf];
          tc_fence_after();
          const uint32_t ga = smem_u32(sG + buf * kGBytes), xb = smem_u32(sXt);
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < D / 8; ++kk) {
              const uint32_t koff = (uint32_t)(kk >> 2) * (D * 128) + (uint32_t)(kk & 3) * 32;
              const uint32_t xoff = (uint32_t)(kk >> 2) * (32 * 128) + (uint32_t)(kk & 3) * 32;
              mma_tf32_ss(tmem_d, sdesc(ga + koff, 16, 1024), sdesc(xb + xoff, 16, 1024), idesc,
                          (c > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(bar_mma);
            if (c == CH - 1) mma_commit(bar_seg);
          }
          __syncwarp();
          if (!mbar_wait_warp(bar_mma, (uint32_t)(n & 1))) {
            ok = false;
            break;
          }
        }
      }
      if (!ok) {
        if (elect_one()) {
          for (int bf = 0; bf < 2; ++bf)
            if (g_iss[bf] > g_cons[bf]) drain_wait(&bar_g[bf], (uint32_t)((g_iss[bf] - 1) & 1));
        }
        __syncwarp();
      }
    }
  } else {
    const int r = tid;
    float x[32];
    if (dM_out) {
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const float4 t = *reinterpret_cast<const float4*>(dM_out + ((size_t)bh * D + r) * D + c0 + e);
        x[e] = t.x; x[e + 1] = t.y; x[e + 2] = t.z; x[e + 3] = t.w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) x[e] = 0.f;
    }
    // GM of the next segment in the sequence (the sum of its query tiles' partials, in
    // tile order), loaded while the current one is used
    float nx[32];
    auto load_gm = [&](int s) {
#pragma unroll
      for (int e = 0; e < 32; ++e) nx[e] = 0.f;
      const float* src = GMp + (((size_t)bh * S + s) * T * D + r) * D + c0;
      for (int t = 0; t < T; ++t, src += (size_t)D * D) {
        float4 v4[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v4[e] = __ldg(reinterpret_cast<const float4*>(src + 4 * e));
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          nx[4 * e] += v4[e].x; nx[4 * e + 1] += v4[e].y;
          nx[4 * e + 2] += v4[e].z; nx[4 * e + 3] += v4[e].w;
        }
      }
    };
    if (S > 0) load_gm(S - 1);
    for (int q = 0; q < S; ++q) {
      const int s = S - 1 - q;
      {  // dM_s -> hi / lo bf16
        __nv_bfloat16* hi = dMs + ((size_t)bh * S + s) * 2 * D * D + (size_t)r * D + c0;
        __nv_bfloat16* lo = hi + D * D;
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint32_t h4[4], l4[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const __nv_bfloat162 hv = __floats2bfloat162_rn(x[e + 2 * t], x[e + 2 * t + 1]);
            const float2 hf = __bfloat1622float2(hv);
            const __nv_bfloat162 lv = __floats2bfloat162_rn(x[e + 2 * t] - hf.x, x[e + 2 * t + 1] - hf.y);
            h4[t] = *reinterpret_cast<const uint32_t*>(&hv);
            l4[t] = *reinterpret_cast<const uint32_t*>(&lv);
          }
          *reinterpret_cast<uint4*>(hi + e) = make_uint4(h4[0], h4[1], h4[2], h4[3]);
          *reinterpret_cast<uint4*>(lo + e) = make_uint4(l4[0], l4[1], l4[2], l4[3]);
        }
      }
      float gm[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) gm[e] = nx[e];
      if (s > 0) load_gm(s - 1);
      if (delta) {
        // X^T block (tf32) -> shared memory: row c, K-major, 4 boxes of 32 k
        const uint32_t kb = (uint32_t)(r >> 5), kin = (uint32_t)(r & 31);
#pragma unroll
        for (int cc = 0; cc < 32; ++cc) {
          const uint32_t off = kb * (32 * 128) + sw128((uint32_t)cc, kin >> 2) + (kin & 3) * 4;
          *reinterpret_cast<uint32_t*>(sXt + off) = tf32_rna(x[cc]);
        }
        fence_proxy_async_smem();
        mbar_arrive_warp(bar_xt);
        if (!mbar_wait_warp(bar_seg, (uint32_t)(q & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t gx[32];
        tmem_ld32(tmem_d + ((uint32_t)(warp * 32) << 16), gx);
        tmem_wait_ld();
        tc_fence_before();
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] += gm[e] - __uint_as_float(gx[e]);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] += gm[e];
      }
    }
    if (dM_in && ok) {
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(dM_in + ((size_t)bh * D + r) * D + c0 + e) =
            make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_d, 32);
  }
}

// ---------------------------------------------------------------------------
// dz: grid = BH, block 128 (feature t). dz_s for s = S-1 .. 0, then dz_in.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(D)
dz_bwd_kernel(const float* __restrict__ Gzp, const float* __restrict__ gzk, const float* dz_out,
              float* __restrict__ dzs, float* dz_in, int S, int T, int mode) {
  const int bh = blockIdx.x, t = threadIdx.x;
  float x = dz_out ? dz_out[(size_t)bh * D + t] : 0.f;
  for (int s = S - 1; s >= 0; --s) {
    dzs[((size_t)bh * S + s) * D + t] = x;
    for (int jj = 0; jj < T; ++jj) x += Gzp[(((size_t)bh * S + s) * T + jj) * D + t];
    if (mode == 1)
      for (int jj = 0; jj < T; ++jj) x += gzk[(((size_t)bh * S + s) * T + jj) * D + t];
  }
  if (dz_in) dz_in[(size_t)bh * D + t] = x;
}

// ---------------------------------------------------------------------------
// The two attention kernels below share one pipeline. Every 128-wide key (dq) or
// query (dk/dv) tile is taken as two 64-column halves, h = 2 n + a for load n and
// half a, alternating between two tensor-memory buffers (scores and dP' side by
// side, 64 fp32 columns each). Warpgroup a (warps 4a .. 4a+3) does the softmax
// arithmetic of every half a, so while one warpgroup works on half h the tensor
// cores compute half h + 1 (and the gradient products of half h - 1). Warp 8 is the
// TMA producer, warp 9 allocates tensor memory and issues every MMA from one
// elected lane. Barriers: SFULL[b] (scores of a half in buffer b ready, one
// tcgen05.commit), PFULL[b] (the warpgroup is done with the buffer: its values read
// and, where a product follows, the half's bf16 operand written over them; four warp
// arrivals); each completes once per use of its buffer and cannot run a phase ahead
// of its waiter (the next use of a buffer is issued only after the previous one's
// PFULL, and its PFULL needs the next SFULL). tests/test_pipeline_model.py checks
// these protocols on the CPU.
// ---------------------------------------------------------------------------
constexpr int kPipeThreads = 320;
constexpr uint32_t kIdN64 = idesc_f32acc(1, 0, 0, 128, 64);

// D = A B^T with N = 64: A[m][k] a full tile, B the 64 rows starting at row 64 a of
// a tile (both K-major, K = 128)
__device__ __forceinline__ void gemm_kk_n64(uint32_t d, const uint8_t* a, const uint8_t* b_tile,
                                            int half) {
  const uint32_t sa = smem_u32(a), sb = smem_u32(b_tile) + (uint32_t)half * 64 * 128;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    mma_bf16_ss(d, kdesc(sa, kk), kdesc(sb, kk), kIdN64, kk > 0 ? 1u : 0u);
}
// D (+)= A X with K = 64: A in tensor memory (32 columns of bf16 pairs), X the 64 rows
// starting at row 64 a of a tile (MN-major, N = 128)
__device__ __forceinline__ void gemm_tm_k64(uint32_t d, uint32_t ta, const uint8_t* x_tile,
                                            int half, bool acc) {
  const uint32_t sx = smem_u32(x_tile) + (uint32_t)half * 64 * 128;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
    mma_bf16_ts(d, ta + 8 * kk, mdesc(sx, kk), kIdKM, (acc || kk > 0) ? 1u : 0u);
}

enum {
  P_ONCE = 0,     // tiles loaded once (Q/dout or K/V)
  P_FULL = 1,     // [2] ring stage loaded
  P_FREE = 3,     // [2] ring stage no longer read by the tensor cores
  P_SFULL = 5,    // [2]
  P_PFULL = 7,    // [2]
  P_DONE = 9,     // every MMA finished
  P_COUNT = 10
};

// the epilogue's steps: memory-path tiles loaded, operand written by the softmax
// warps (8 warp arrivals), products done
enum { P_X = P_COUNT, P_SK, P_M1, P_SK2, P_M2, P_COUNT2 };

__device__ __forceinline__ void pipe_init(uint64_t* bars) {
  for (int x = 0; x < P_COUNT2; ++x) {
    uint32_t c = 1;
    if (x == P_PFULL || x == P_PFULL + 1) c = 4;
    if (x == P_SK || x == P_SK2) c = 8;
    mbar_init(&bars[x], c);
  }
  fence_barrier_init();
}

// ---------------------------------------------------------------------------
// dq: grid = BH * S * T, one CTA per query tile i. Loads n = 0 .. 2 (i+1) - 1 stream
// the key tiles j = n mod (i+1) through a 2-stage K/V ring, twice: the first sweep
// gives each row's log-sum-exp and D' = dout . A_dot (a running maximum, sum and
// dP'-weighted sum per warpgroup, merged once), the second dS and dQ = sum dS K.
// Tensor memory: buffer 0 [0, 128), buffer 1 [128, 256), dQ [256, 384).
// After the loop the same CTA runs the retrieval's backward for its query rows,
// with Q and dout still in shared memory and M_{s-1} (bf16 hi) loaded into the K
// ring stage that frees first: sigma(Q) replaces Q, num = sigma(Q) M -> buffer 0,
// dnum = g dout / den over the other K stage, dden = -rowsum(g dout * A_mem) / den
// as a 129th column right after it; dsigma(Q) = dnum M^T -> [384, 512) and
// sigma(Q)^T [dnum | dden] (N = 144) -> [0, 144), the tile's GM and Gz partials.
// dq = dQ + (dsigma(Q) + dden z) * sigma'(Q) is written once, in bf16.
// ---------------------------------------------------------------------------
constexpr int kDqSmem = 6 * kTile + 3 * 2 * D * 4 + 64 + D * 4 + 256 + 1024;

__global__ void __launch_bounds__(kPipeThreads, 1)
dq_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ CUtensorMap tm_m, const float* __restrict__ beta,
              const float* __restrict__ zprev, float* __restrict__ lse_out,
              float* __restrict__ dp_out, float* __restrict__ dot_part,
              float* __restrict__ mem_part, float* __restrict__ GMp, float* __restrict__ Gzp,
              __nv_bfloat16* __restrict__ dq, const BwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sDO = smem + kTile;
  uint8_t* sK = smem + 2 * kTile;  // 2 stages
  uint8_t* sV = smem + 4 * kTile;  // 2 stages
  float* xs = reinterpret_cast<float*>(smem + 6 * kTile);  // [wg][m | l | dacc][128]
  float* red = xs + 3 * 2 * D;
  float* sZ = red + 16;                                     // z_{s-1}
  uint64_t* bars = reinterpret_cast<uint64_t*>(sZ + D);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + P_COUNT2);
  uint8_t* sM = sK;           // M_{s-1} (hi): K stage 0, free once load nl - 2 is done
  uint8_t* sDN = sK + kTile;  // dnum: K stage 1; dden in the next 64-column box (V stage 0)

  // tiles of a segment are adjacent in the grid (K/V stay in L2), the heaviest first
  int bh, s, i;
  decode3(p, blockIdx.x, bh, s, i);
  i = p.T - 1 - i;
  const unsigned tile = (unsigned)((bh * p.S + s) * p.T + i);  // index of the partials
  const int b = bh / p.H, h = bh - b * p.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = i + 1, nl = 2 * nk, nh = 2 * nl;
  const int row0 = s * p.N + i * 128;
  if (threadIdx.x == 0) pipe_init(bars);
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot, tQ = tmem + 256;
  bool ok = true;

  if (warp == 8) {
    // ---------------- producer ----------------
    if (lane == 0) {
      int iss[2] = {0, 0};
      mbar_arrive_expect_tx(&bars[P_ONCE], 2 * kTile);
      load_rows(sQ, &tm_q, &bars[P_ONCE], row0, h, b);
      load_rows(sDO, &tm_do, &bars[P_ONCE], row0, h, b);
      for (int n = 0; n < nl; ++n) {
        const int st = n & 1, j = n % nk;
        if (n >= 2 && !mbar_wait(&bars[P_FREE + st], (uint32_t)(((n >> 1) - 1) & 1))) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&bars[P_FULL + st], 2 * kTile);
        load_rows(sK + st * kTile, &tm_k, &bars[P_FULL + st], s * p.N + j * 128, h, b);
        load_rows(sV + st * kTile, &tm_v, &bars[P_FULL + st], s * p.N + j * 128, h, b);
        ++iss[st];
      }
      // K stage 0 was last used by load nl - 2 (nl is even)
      bool x_iss = false;
      if (ok && !mbar_wait(&bars[P_FREE], (uint32_t)(((nl - 2) >> 1) & 1))) ok = false;
      if (ok) {
        mbar_arrive_expect_tx(&bars[P_X], kTile + D * 4);
        load_plane(sM, &tm_m, &bars[P_X], (bh * p.S + s) * 2);
        bulk_load(sZ, zprev + ((size_t)bh * p.S + s) * D, D * 4, &bars[P_X]);
        x_iss = true;
      }
      if (!ok) {
        drain_wait(&bars[P_ONCE], 0);
        for (int st = 0; st < 2; ++st)
          if (iss[st] > 0) drain_wait(&bars[P_FULL + st], (uint32_t)((iss[st] - 1) & 1));
        if (x_iss) drain_wait(&bars[P_X], 0);
      }
    }
  } else if (warp == 9) {
    // ---------------- MMA issuer ----------------
    auto issue_sdp = [&](int hh) -> bool {
      const int n = hh >> 1, a = hh & 1, st = n & 1;
      if (a == 0 && !mbar_wait_warp(&bars[P_FULL + st], (uint32_t)((n >> 1) & 1))) return false;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t tb = tmem + (uint32_t)a * 128;
        gemm_kk_n64(tb, sQ, sK + st * kTile, a);        // S  = Q K_j[64a..]^T
        gemm_kk_n64(tb + 64, sDO, sV + st * kTile, a);  // dP' = dout V_j[64a..]^T
        mma_commit(&bars[P_SFULL + a]);
        if (n < nk && a == 1) mma_commit(&bars[P_FREE + st]);  // first sweep: done with K/V
      }
      __syncwarp();
      return true;
    };
    ok = mbar_wait_warp(&bars[P_ONCE], 0) && issue_sdp(0) && issue_sdp(1);
    for (int hh = 0; ok && hh < nh; ++hh) {
      const int n = hh >> 1, a = hh & 1, st = n & 1;
      if (!mbar_wait_warp(&bars[P_PFULL + a], (uint32_t)(n & 1))) {
        ok = false;
        break;
      }
      if (n >= nk) {
        tc_fence_after();
        if (elect_one()) {
          // dQ += dS_h K_j[64a..]  (dS in the first 32 columns of the buffer)
          gemm_tm_k64(tQ, tmem + (uint32_t)a * 128, sK + st * kTile, a, n > nk || a == 1);
          if (a == 1) mma_commit(&bars[P_FREE + st]);
        }
        __syncwarp();
      }
      if (hh + 2 < nh && !issue_sdp(hh + 2)) ok = false;
    }
    if (elect_one()) mma_commit(&bars[P_DONE]);
    __syncwarp();
    // the retrieval's backward
    ok = ok && mbar_wait_warp(&bars[P_X], 0) && mbar_wait_warp(&bars[P_SK], 0);
    if (ok) {
      tc_fence_after();
      if (elect_one()) {
        gemm_km(tmem, sQ, sM, false);  // num = sigma(Q) M
        mma_commit(&bars[P_M1]);
      }
      __syncwarp();
      ok = mbar_wait_warp(&bars[P_SK2], 0);
    }
    if (ok) {
      tc_fence_after();
      if (elect_one()) {
        gemm_kk(tmem + 384, sDN, sM, false);  // dsigma(Q) = dnum M^T
        // [GM | Gz] = sigma(Q)^T [dnum | dden]: both operands MN-major, N = 144
        const uint32_t sa = smem_u32(sQ), sb = smem_u32(sDN);
        constexpr uint32_t kIdG = idesc_f32acc(1, 1, 1, 128, 144);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16_ss(tmem, mdesc(sa, kk), mdesc(sb, kk), kIdG, kk > 0 ? 1u : 0u);
        mma_commit(&bars[P_M2]);
      }
      __syncwarp();
    }
    if (!ok) {
      if (elect_one()) mma_commit(&bars[P_M2]);
      __syncwarp();
      drain_wait(&bars[P_M2], 0);
    }
  } else {
    // ---------------- softmax warpgroups ----------------
    const int wg = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tb = tmem + (uint32_t)wg * 128 + lane_off;
    const float g = 1.f / (1.f + expf(-beta[h]));
    const float cds = (1.f - g) * p.rsd, sl = p.sl;
    float m = -INFINITY, l = 0.f, dacc = 0.f;
    for (int n = 0; ok && n < nk; ++n) {
      if (!mbar_wait_warp(&bars[P_SFULL + wg], (uint32_t)(n & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool diag = n == i;
      uint32_t sv[64], pv[64];
      tmem_ld32(tb, *reinterpret_cast<uint32_t(*)[32]>(sv));
      tmem_ld32(tb + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
      tmem_ld32(tb + 64, *reinterpret_cast<uint32_t(*)[32]>(pv));
      tmem_ld32(tb + 96, *reinterpret_cast<uint32_t(*)[32]>(pv + 32));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive_warp(&bars[P_PFULL + wg]);  // the buffer may take the next half
      float* sf = reinterpret_cast<float*>(sv);
      if (diag) {  // keys after the row do not count
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (64 * wg + c > r) sf[c] = -INFINITY;
      }
      float mx8[8];
#pragma unroll
      for (int q8 = 0; q8 < 8; ++q8)
        mx8[q8] = fmaxf(fmax3(sf[q8], sf[8 + q8], sf[16 + q8]),
                        fmax3(sf[24 + q8], sf[32 + q8], fmax3(sf[40 + q8], sf[48 + q8], sf[56 + q8])));
      const float mx = fmaxf(fmax3(mx8[0], mx8[1], mx8[2]),
                             fmaxf(fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      if (mx == -INFINITY) continue;  // every key of this half is after the row
      const float mn = fmaxf(m, mx);
      const float alpha = ex2_approx((m - mn) * sl);  // 0 while m = -inf
      const float mb = mn * sl;
      float la[4] = {0.f, 0.f, 0.f, 0.f}, da[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float pe = ex2_approx(fmaf(sf[c], sl, -mb));  // 0 where masked (-inf)
        la[c & 3] += pe;
        da[c & 3] = fmaf(pe, __uint_as_float(pv[c]), da[c & 3]);
      }
      l = fmaf(l, alpha, (la[0] + la[1]) + (la[2] + la[3]));
      dacc = fmaf(dacc, alpha, (da[0] + da[1]) + (da[2] + da[3]));
      m = mn;
    }
    // merge the two warpgroups' running statistics of row r
    if (ok) {
      xs[(wg * 3 + 0) * D + r] = m;
      xs[(wg * 3 + 1) * D + r] = l;
      xs[(wg * 3 + 2) * D + r] = dacc;
    }
    named_bar_sync(1, 256);
    float lse2 = 0.f, dpv = 0.f;
    {
      const float m0 = xs[0 * D + r], l0 = xs[1 * D + r], d0 = xs[2 * D + r];
      const float m1 = xs[3 * D + r], l1 = xs[4 * D + r], d1 = xs[5 * D + r];
      const float mt = fmaxf(m0, m1);
      const float e0 = ex2_approx((m0 - mt) * sl), e1 = ex2_approx((m1 - mt) * sl);
      const float lt = l0 * e0 + l1 * e1;
      lse2 = mt * sl + log2f(lt);
      dpv = (d0 * e0 + d1 * e1) / lt;
    }
    for (int n = nk; ok && n < nl; ++n) {
      if (!mbar_wait_warp(&bars[P_SFULL + wg], (uint32_t)(n & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sv[64], pv[64], pk[32];
      tmem_ld32(tb, *reinterpret_cast<uint32_t(*)[32]>(sv));
      tmem_ld32(tb + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
      tmem_ld32(tb + 64, *reinterpret_cast<uint32_t(*)[32]>(pv));
      tmem_ld32(tb + 96, *reinterpret_cast<uint32_t(*)[32]>(pv + 32));
      tmem_wait_ld();
      float* sf = reinterpret_cast<float*>(sv);
      if (n == nl - 1) {  // the diagonal tile: keys after the row get P = 0
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (64 * wg + c > r) sf[c] = -INFINITY;
      }
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float p0 = ex2_approx(fmaf(sf[2 * e], sl, -lse2));
        const float p1 = ex2_approx(fmaf(sf[2 * e + 1], sl, -lse2));
        pk[e] = pack_bf16x2(cds * p0 * (__uint_as_float(pv[2 * e]) - dpv),
                            cds * p1 * (__uint_as_float(pv[2 * e + 1]) - dpv));
      }
      // dS over the first 32 columns of the buffer: scores this thread has read
      tmem_st32_(tb, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive_warp(&bars[P_PFULL + wg]);
    }
    // ---- the retrieval's backward (every product of the loop done: Q may change) ----
    ok = ok && mbar_wait_warp(&bars[P_DONE], 0) && mbar_wait_warp(&bars[P_X], 0);
    float denp = 0.f;
    if (ok) {
#pragma unroll
      for (int u = 8 * wg; u < 8 * wg + 8; ++u) {
        float f[8];
        unpack8(ld_unit(sQ, r, u), f);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          f[e] = sig(f[e]);
          denp = fmaf(f[e], sZ[8 * u + e], denp);
        }
        st_unit(sQ, r, u, f);  // sigma(Q) over Q
      }
    }
    fence_proxy_async_smem();
    xs[wg * D + r] = denp;
    named_bar_sync(1, 256);
    const float den = xs[r] + xs[D + r];
    const float inv = den != 0.f ? 1.f / den : 0.f;
    tc_fence_before();
    mbar_arrive_warp(&bars[P_SK]);
    float dd = 0.f, memt = 0.f;
    ok = ok && mbar_wait_warp(&bars[P_M1], 0);
    if (ok) {
      tc_fence_after();
      uint32_t nv[64];
      tmem_ld32(tmem + lane_off + 64 * wg, *reinterpret_cast<uint32_t(*)[32]>(nv));
      tmem_ld32(tmem + lane_off + 64 * wg + 32, *reinterpret_cast<uint32_t(*)[32]>(nv + 32));
      tmem_wait_ld();
#pragma unroll
      for (int u8 = 0; u8 < 8; ++u8) {
        const int u = 8 * wg + u8;
        float o[8], dn[8];
        unpack8(ld_unit(sDO, r, u), o);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float am = __uint_as_float(nv[8 * u8 + e]) * inv;  // A_mem
          const float da = g * o[e];
          dn[e] = da * inv;
          dd = fmaf(da, am, dd);
          memt = fmaf(o[e], am, memt);
        }
        st_unit(sDN, r, u, dn);
      }
    }
    xs[wg * D + r] = dd;  // every thread has read den above (P_M1 needs all P_SK arrivals)
    named_bar_sync(1, 256);
    const float dden = -(xs[r] + xs[D + r]) * inv;
    if (wg == 0) {
      // columns 128 and 129 of the product's right operand, (row r, columns 0 and 1) of
      // box 2: dden as a bf16 pair hi + lo, so that Gz keeps fp32 accuracy in dden
      const __nv_bfloat16 hi = __float2bfloat16_rn(dden);
      const __nv_bfloat16 lo = __float2bfloat16_rn(dden - __bfloat162float(hi));
      __nv_bfloat162 pr;
      pr.x = hi;
      pr.y = lo;
      *reinterpret_cast<__nv_bfloat162*>(sDN + 2 * kSub + sw128((uint32_t)r, 0)) = pr;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive_warp(&bars[P_SK2]);
    ok = ok && mbar_wait_warp(&bars[P_M2], 0);
    const size_t rowi = (size_t)bh * p.L + row0 + r;
    if (ok) {
      tc_fence_after();
      __nv_bfloat16* dst = dq + rowi * D;
      float* gm = GMp + ((size_t)tile * D + r) * D;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const uint32_t col = 64 * wg + 32 * c;
        uint32_t qv[32], sv[32], gv[32];
        tmem_ld32(tQ + lane_off + col, qv);
        tmem_ld32(tmem + 384 + lane_off + col, sv);
        tmem_ld32(tmem + lane_off + col, gv);
        tmem_wait_ld();
#pragma unroll
        for (int u4 = 0; u4 < 4; ++u4) {
          const int u = (int)(col >> 3) + u4;
          float sq[8], o[8];
          unpack8(ld_unit(sQ, r, u), sq);  // sigma(Q), bf16
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float dsq = fmaf(dden, sZ[8 * u + e], __uint_as_float(sv[8 * u4 + e]));
            o[e] = fmaf(dsq, fminf(sq[e], 1.f), __uint_as_float(qv[8 * u4 + e]));  // sigma' = min(sigma, 1)
          }
          *reinterpret_cast<uint4*>(dst + 8 * u) =
              make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                         pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
        }
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(gm + col + e) =
              make_float4(__uint_as_float(gv[e]), __uint_as_float(gv[e + 1]),
                          __uint_as_float(gv[e + 2]), __uint_as_float(gv[e + 3]));
      }
      if (wg == 0) {
        uint32_t zv[32];
        tmem_ld32(tmem + lane_off + 128, zv);  // columns 128, 129: sigma(Q)^T dden (hi, lo)
        tmem_wait_ld();
        Gzp[(size_t)tile * D + r] = __uint_as_float(zv[0]) + __uint_as_float(zv[1]);
        lse_out[rowi] = lse2;
        dp_out[rowi] = dpv;
      }
    }
    // the tile's sums of D' and of dout * A_mem (for dbeta); every softmax thread
    // reaches the barrier, whatever its waits returned
    {
      float t0 = (ok && wg == 0) ? dpv : 0.f, t1 = ok ? memt : 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        t0 += __shfl_xor_sync(0xffffffffu, t0, o);
        t1 += __shfl_xor_sync(0xffffffffu, t1, o);
      }
      if (lane == 0) {
        red[warp] = t0;
        red[8 + warp] = t1;
      }
      named_bar_sync(2, 256);
      if (threadIdx.x == 0 && ok) {
        float a0 = 0.f, a1 = 0.f;
        for (int w = 0; w < 8; ++w) {
          a0 += red[w];
          a1 += red[8 + w];
        }
        dot_part[tile] = a0;
        mem_part[tile] = a1;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// dkdv: grid = BH * S * T, one CTA per key tile j. Loads n = 0 .. T-1-j stream the
// query tiles i = j + n (Q, dout and their rows' statistics) through a 2-stage ring.
// Half a of load n is queries [64a, 64a + 64): S^T = K_j Q^T and dP'^T = V_j dout^T
// (128 keys x 64 queries), then dV += (1-g) P^T dout and dK += dS^T Q over those 64
// queries. Tensor memory: buffer 0 [0, 128), buffer 1 [128, 256), dV, dK.
// After the loop the same CTA runs the memory update's backward for its key rows,
// with K and V still in shared memory and dM_s (bf16, the reverse chain's stack)
// loaded into the ring stage that frees first: sigma(K) replaces K in place, and
//   Linear: dV += sigma(K) dM_s;  dsigma(K) = V dM_s^T (+ dz_s)
//   Delta:  R = sigma(K) M_{s-1} / den_K, dU = sigma(K) dM_s, dV += dU, U = V - R
//           (over V), dnumR = -dU / den_K, ddenR = rowsum(dU * R) / den_K,
//           dsigma(K) = U dM_s^T + dnumR M^T + ddenR z, and the tile's sigma(K)^T ddenR
//           for the z gradients (dz_s, which needs every later segment's, is added
//           to dk by dk_dz_kernel afterwards).
// ---------------------------------------------------------------------------
constexpr int kDkdvSmem = 6 * kTile + 2 * 2 * D * 4 + 5 * D * 4 + 64 + 256 + 1024;

__global__ void __launch_bounds__(kPipeThreads, 1)
dkdv_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const __grid_constant__ CUtensorMap tm_m, const __grid_constant__ CUtensorMap tm_x,
                const float* __restrict__ beta, const float* __restrict__ zprev,
                const float* __restrict__ lse, const float* __restrict__ dpr,
                const float* __restrict__ dzs, float* __restrict__ gzk,
                __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv, const BwdParams p,
                int mode) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sV = smem + kTile;
  uint8_t* sQ = smem + 2 * kTile;   // 2 stages
  uint8_t* sDO = smem + 4 * kTile;  // 2 stages
  float* sLD = reinterpret_cast<float*>(smem + 6 * kTile);  // [stage][lse | D'][128]
  float* xs = sLD + 4 * D;    // [2][128] per-warpgroup partial row sums
  float* sDD = xs + 2 * D;    // [128] ddenR
  float* gzp = sDD + D;       // [2][128] partial column sums
  uint64_t* bars = reinterpret_cast<uint64_t*>(gzp + 2 * D + 16);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + P_COUNT2);

  int bh, s, j;
  decode3(p, blockIdx.x, bh, s, j);
  const int b = bh / p.H, h = bh - b * p.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nl = p.T - j, nh = 2 * nl;
  const int krow = s * p.N + j * 128;
  const bool delta = mode == 1;
  const int sx = nl & 1;  // ring stage that holds dM_s (and M_{s-1}, z_{s-1}) at the end
  uint8_t* sX = sQ + sx * kTile;         // dM_s (hi)
  uint8_t* sMp = sDO + sx * kTile;       // M_{s-1} (hi), Delta
  uint8_t* sDN = sQ + (sx ^ 1) * kTile;  // dnumR, Delta (the last load's stage)
  const float* sZ = sLD + sx * 2 * D;    // z_{s-1}, Delta
  if (threadIdx.x == 0) {
    pipe_init(bars);
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot, tV = tmem + 256, tK = tmem + 384;
  bool ok = true;

  if (warp == 8) {
    if (lane == 0) {
      int iss[2] = {0, 0};
      bool x_iss = false;
      mbar_arrive_expect_tx(&bars[P_ONCE], 2 * kTile);
      load_rows(sK, &tm_k, &bars[P_ONCE], krow, h, b);
      load_rows(sV, &tm_v, &bars[P_ONCE], krow, h, b);
      for (int n = 0; n < nl; ++n) {
        const int st = n & 1, rq = s * p.N + (j + n) * 128;
        if (n >= 2 && !mbar_wait(&bars[P_FREE + st], (uint32_t)(((n >> 1) - 1) & 1))) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&bars[P_FULL + st], 2 * kTile + 2 * D * 4);
        load_rows(sQ + st * kTile, &tm_q, &bars[P_FULL + st], rq, h, b);
        load_rows(sDO + st * kTile, &tm_do, &bars[P_FULL + st], rq, h, b);
        bulk_load(sLD + st * 2 * D, lse + (size_t)bh * p.L + rq, D * 4, &bars[P_FULL + st]);
        bulk_load(sLD + st * 2 * D + D, dpr + (size_t)bh * p.L + rq, D * 4, &bars[P_FULL + st]);
        ++iss[st];
      }
      // stage sx was last used by load nl - 2 (never when nl == 1)
      if (ok && nl >= 2 && !mbar_wait(&bars[P_FREE + sx], (uint32_t)(((nl - 2) >> 1) & 1)))
        ok = false;
      if (ok) {
        const int plane = (bh * p.S + s) * 2;
        mbar_arrive_expect_tx(&bars[P_X], delta ? 2 * kTile + D * 4 : kTile);
        load_plane(sX, &tm_x, &bars[P_X], plane);
        if (delta) {
          load_plane(sMp, &tm_m, &bars[P_X], plane);
          bulk_load(sLD + sx * 2 * D, zprev + ((size_t)bh * p.S + s) * D, D * 4, &bars[P_X]);
        }
        x_iss = true;
      }
      if (!ok) {
        drain_wait(&bars[P_ONCE], 0);
        for (int st = 0; st < 2; ++st)
          if (iss[st] > 0) drain_wait(&bars[P_FULL + st], (uint32_t)((iss[st] - 1) & 1));
        if (x_iss) drain_wait(&bars[P_X], 0);
      }
    }
  } else if (warp == 9) {
    auto issue_sdp = [&](int hh) -> bool {
      const int n = hh >> 1, a = hh & 1, st = n & 1;
      if (a == 0 && !mbar_wait_warp(&bars[P_FULL + st], (uint32_t)((n >> 1) & 1))) return false;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t tb = tmem + (uint32_t)a * 128;
        gemm_kk_n64(tb, sK, sQ + st * kTile, a);        // S^T  = K_j Q[64a..]^T
        gemm_kk_n64(tb + 64, sV, sDO + st * kTile, a);  // dP'^T = V_j dout[64a..]^T
        mma_commit(&bars[P_SFULL + a]);
      }
      __syncwarp();
      return true;
    };
    ok = mbar_wait_warp(&bars[P_ONCE], 0) && issue_sdp(0) && issue_sdp(1);
    for (int hh = 0; ok && hh < nh; ++hh) {
      const int n = hh >> 1, a = hh & 1, st = n & 1;
      if (!mbar_wait_warp(&bars[P_PFULL + a], (uint32_t)(n & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (elect_one()) {
        const uint32_t tb = tmem + (uint32_t)a * 128;
        gemm_tm_k64(tV, tb, sDO + st * kTile, a, hh > 0);      // dV += (1-g) P^T dout
        gemm_tm_k64(tK, tb + 64, sQ + st * kTile, a, hh > 0);  // dK += dS^T Q
        if (a == 1) mma_commit(&bars[P_FREE + st]);
      }
      __syncwarp();
      if (hh + 2 < nh && !issue_sdp(hh + 2)) ok = false;
    }
    if (elect_one()) mma_commit(&bars[P_DONE]);
    __syncwarp();
    // the memory update's backward: sigma(K) written over K, dM_s (and M, z) loaded
    ok = ok && mbar_wait_warp(&bars[P_X], 0) && mbar_wait_warp(&bars[P_SK], 0);
    if (ok) {
      tc_fence_after();
      if (elect_one()) {
        if (delta) {
          gemm_km(tmem, sK, sMp, false);       // R_num = sigma(K) M_{s-1}
          gemm_km(tmem + 128, sK, sX, false);  // dU = sigma(K) dM_s
        } else {
          gemm_kk(tmem, sV, sX, false);        // V dM_s^T
        }
        gemm_km(tV, sK, sX, true);             // dV += sigma(K) dM_s
        mma_commit(&bars[P_M1]);
      }
      __syncwarp();
      if (delta) {
        ok = mbar_wait_warp(&bars[P_SK2], 0);
        if (ok) {
          tc_fence_after();
          if (elect_one()) {
            gemm_kk(tmem, sV, sX, false);     // U dM_s^T   (U written over V)
            gemm_kk(tmem, sDN, sMp, true);    // + dnumR M^T
            mma_commit(&bars[P_M2]);
          }
          __syncwarp();
        }
      }
    }
    if (!ok) {
      if (elect_one()) mma_commit(&bars[P_M2]);
      __syncwarp();
      drain_wait(&bars[P_M2], 0);
    }
  } else {
    const int wg = warp >> 2;
    const int r = (warp & 3) * 32 + lane;  // key row of the tile
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tb = tmem + (uint32_t)wg * 128 + lane_off;
    const float g = 1.f / (1.f + expf(-beta[h]));
    const float cp = 1.f - g, cds = (1.f - g) * p.rsd, sl = p.sl;
    for (int n = 0; ok && n < nl; ++n) {
      const int st = n & 1;
      // the stage's row statistics (written by TMA) and this half's scores
      if (!mbar_wait_warp(&bars[P_FULL + st], (uint32_t)((n >> 1) & 1)) ||
          !mbar_wait_warp(&bars[P_SFULL + wg], (uint32_t)(n & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* ls = sLD + st * 2 * D + 64 * wg;
      const float* dps = ls + D;
      uint32_t sv[64], pv[64], pk1[32], pk2[32];
      tmem_ld32(tb, *reinterpret_cast<uint32_t(*)[32]>(sv));
      tmem_ld32(tb + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
      tmem_ld32(tb + 64, *reinterpret_cast<uint32_t(*)[32]>(pv));
      tmem_ld32(tb + 96, *reinterpret_cast<uint32_t(*)[32]>(pv + 32));
      tmem_wait_ld();
      float* sf = reinterpret_cast<float*>(sv);
      if (n == 0) {  // the diagonal tile: queries before key r get P = 0
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (64 * wg + c < r) sf[c] = -INFINITY;
      }
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float2 lq = *reinterpret_cast<const float2*>(ls + 2 * e);
        const float2 dq2 = *reinterpret_cast<const float2*>(dps + 2 * e);
        const float p0 = ex2_approx(fmaf(sf[2 * e], sl, -lq.x));
        const float p1 = ex2_approx(fmaf(sf[2 * e + 1], sl, -lq.y));
        pk1[e] = pack_bf16x2(cp * p0, cp * p1);
        pk2[e] = pack_bf16x2(cds * p0 * (__uint_as_float(pv[2 * e]) - dq2.x),
                             cds * p1 * (__uint_as_float(pv[2 * e + 1]) - dq2.y));
      }
      // P^T and dS^T over the first 32 columns of the scores and of dP'^T (read)
      tmem_st32_(tb, pk1);
      tmem_st32_(tb + 64, pk2);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive_warp(&bars[P_PFULL + wg]);
    }
    // ---- the memory update's backward ----
    // every MMA of the loop is done (K may be overwritten); z_{s-1} is needed for Delta
    ok = ok && mbar_wait_warp(&bars[P_DONE], 0) && (!delta || mbar_wait_warp(&bars[P_X], 0));
    float denp = 0.f;
    if (ok) {
#pragma unroll
      for (int u = 8 * wg; u < 8 * wg + 8; ++u) {
        float f[8];
        unpack8(ld_unit(sK, r, u), f);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          f[e] = sig(f[e]);
          if (delta) denp = fmaf(f[e], sZ[8 * u + e], denp);
        }
        st_unit(sK, r, u, f);
      }
    }
    fence_proxy_async_smem();
    xs[wg * D + r] = denp;
    named_bar_sync(1, 256);
    const float denK = xs[r] + xs[D + r];
    tc_fence_before();
    mbar_arrive_warp(&bars[P_SK]);
    const size_t rowk = (size_t)bh * p.L + krow + r;
    float ddenR = 0.f;
    if (delta) {
      ok = ok && mbar_wait_warp(&bars[P_M1], 0);
      float ddp = 0.f;
      if (ok) {
        tc_fence_after();
        const float inv = denK != 0.f ? 1.f / denK : 0.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t rn[32], du[32];
          tmem_ld32(tmem + lane_off + 64 * wg + 32 * c, rn);
          tmem_ld32(tmem + 128 + lane_off + 64 * wg + 32 * c, du);
          tmem_wait_ld();
#pragma unroll
          for (int u4 = 0; u4 < 4; ++u4) {
            const int u = 8 * wg + 4 * c + u4;
            float vv[8], uu[8], dn[8];
            unpack8(ld_unit(sV, r, u), vv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float rr = __uint_as_float(rn[8 * u4 + e]) * inv;
              const float dU = __uint_as_float(du[8 * u4 + e]);
              uu[e] = vv[e] - rr;
              dn[e] = -dU * inv;
              ddp = fmaf(dU, rr, ddp);
            }
            st_unit(sV, r, u, uu);   // U over V (this row's V is read)
            st_unit(sDN, r, u, dn);
          }
        }
        ddp *= inv;
      }
      fence_proxy_async_smem();
      xs[wg * D + r] = ddp;
      named_bar_sync(1, 256);
      ddenR = xs[r] + xs[D + r];
      if (wg == 0) sDD[r] = ddenR;
      tc_fence_before();
      mbar_arrive_warp(&bars[P_SK2]);
      named_bar_sync(1, 256);
      {  // sigma(K)^T ddenR over this tile's rows: column r, rows [64 wg, 64 wg + 64)
        float acc = 0.f;
        for (int rr = 64 * wg; rr < 64 * wg + 64; ++rr) acc = fmaf(ld_elem(sK, rr, r), sDD[rr], acc);
        gzp[wg * D + r] = acc;
      }
      named_bar_sync(1, 256);
      if (wg == 0 && ok) gzk[(((size_t)bh * p.S + s) * p.T + j) * D + r] = gzp[r] + gzp[D + r];
      ok = ok && mbar_wait_warp(&bars[P_M2], 0);
    } else {
      ok = ok && mbar_wait_warp(&bars[P_M1], 0);
    }
    if (ok) {
      tc_fence_after();
      const float* dz = dzs + ((size_t)bh * p.S + s) * D;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t a[32], bb[32], xk[32];
        const uint32_t col = 64 * wg + 32 * c;
        tmem_ld32(tV + lane_off + col, a);
        tmem_ld32(tK + lane_off + col, bb);
        tmem_ld32(tmem + lane_off + col, xk);
        tmem_wait_ld();
#pragma unroll
        for (int u4 = 0; u4 < 4; ++u4) {
          const int u = (int)(col >> 3) + u4;
          float sk[8], ov[8], ok8[8];
          unpack8(ld_unit(sK, r, u), sk);  // sigma(K), bf16
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int f = 8 * u + e;
            float dsk = __uint_as_float(xk[8 * u4 + e]);
            dsk = delta ? fmaf(ddenR, sZ[f], dsk) : dsk + dz[f];
            ov[e] = __uint_as_float(a[8 * u4 + e]);
            ok8[e] = fmaf(dsk, fminf(sk[e], 1.f), __uint_as_float(bb[8 * u4 + e]));  // sigma' = min(sigma, 1)
          }
          *reinterpret_cast<uint4*>(dv + rowk * D + 8 * u) =
              make_uint4(pack_bf16x2(ov[0], ov[1]), pack_bf16x2(ov[2], ov[3]),
                         pack_bf16x2(ov[4], ov[5]), pack_bf16x2(ov[6], ov[7]));
          *reinterpret_cast<uint4*>(dk + rowk * D + 8 * u) =
              make_uint4(pack_bf16x2(ok8[0], ok8[1]), pack_bf16x2(ok8[2], ok8[3]),
                         pack_bf16x2(ok8[4], ok8[5]), pack_bf16x2(ok8[6], ok8[7]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Delta: dk += dz_s * sigma'(K), once every segment's z gradient is known.
// grid-stride over the [BH][L][128] elements in units of 8.
__global__ void __launch_bounds__(256)
dk_dz_kernel(const __nv_bfloat16* __restrict__ k, const float* __restrict__ dzs,
             __nv_bfloat16* __restrict__ dk, long long L, int N, int S, long long units) {
  for (long long u = blockIdx.x * (long long)blockDim.x + threadIdx.x; u < units;
       u += (long long)gridDim.x * blockDim.x) {
    const long long row = u >> 4;  // 16 units of 8 per row
    const int f0 = (int)(u & 15) * 8;
    const long long bh = row / L;
    const int s = (int)((row - bh * L) / N);
    const float* dz = dzs + ((size_t)bh * S + s) * D + f0;
    float kf[8], df[8];
    unpack8(*reinterpret_cast<const uint4*>(k + u * 8), kf);
    unpack8(*reinterpret_cast<const uint4*>(dk + u * 8), df);
#pragma unroll
    for (int e = 0; e < 8; ++e) df[e] = fmaf(dz[e], dsig(kf[e]), df[e]);
    *reinterpret_cast<uint4*>(dk + u * 8) =
        make_uint4(pack_bf16x2(df[0], df[1]), pack_bf16x2(df[2], df[3]),
                   pack_bf16x2(df[4], df[5]), pack_bf16x2(df[6], df[7]));
  }
}

// dbeta[h] = g (1 - g) sum over batch rows, segments and query tiles of (sum dout *
// A_mem - sum D'). One warp per head: lane l takes the (batch row, tile) sums l, l+32,
// ... in order, then a fixed shuffle tree (the result does not depend on timing).
__global__ void dbeta_bwd_kernel(const float* __restrict__ beta, const float* __restrict__ mem_part,
                                 const float* __restrict__ dot_part, float* __restrict__ dbeta,
                                 int B, int H, int S, int T) {
  const int h = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (h >= H) return;
  const long long per_b = (long long)S * T, n = (long long)B * per_b;
  double acc = 0.0;
  for (long long x = lane; x < n; x += 32) {
    const long long b = x / per_b, st = x - b * per_b;
    const size_t k = ((size_t)b * H + h) * per_b + st;
    acc += (double)mem_part[k] - (double)dot_part[k];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    const float g = 1.f / (1.f + expf(-beta[h]));
    dbeta[h] = (float)(acc * (double)g * (1.0 - (double)g));
  }
}

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

cudaError_t bf16_bwd_set_attributes() {
  cudaError_t e = cudaFuncSetAttribute(chain_bwd_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kChainSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(dq_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDqSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(dkdv_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kDkdvSmem);
  return e;
}

// Backward scratch after the state path's: per-row statistics, per-query-tile
// partials of the state gradients, the dM_s stack, dz_s, per-tile sums for dbeta.
size_t bf16_bwd_workspace_bytes(int BH, long long L, int S, int T, int CH) {
  const size_t bh = (size_t)BH, rows = bh * (size_t)L, bhs = bh * S;
  return up256(bf16_workspace_bytes(BH, S, CH)) + 2 * up256(rows * 4) +
         up256(bhs * T * D * D * 4) + up256(bhs * T * D * 4) + up256(bhs * 2 * D * D * 2) +
         up256(bhs * D * 4) + up256(bhs * T * D * 4) + 2 * up256(bhs * T * 4);
}

cudaError_t bf16_backward_launch(const __nv_bfloat16* q, const __nv_bfloat16* k,
                                 const __nv_bfloat16* v, const float* beta, const float* M_in,
                                 const float* z_in, const __nv_bfloat16* dout,
                                 const float* dM_out, const float* dz_out, __nv_bfloat16* dq,
                                 __nv_bfloat16* dk, __nv_bfloat16* dv, float* dbeta, float* dM_in,
                                 float* dz_in, int B, int H, long long L, int N, int mode,
                                 void* scratch, int CH, int CL, cudaStream_t stream,
                                 cudaEvent_t const* events) {
  auto mark = [&](int i) {
    if (events && events[i]) cudaEventRecord(events[i], stream);
  };
  const int BH = B * H, S = (int)(L / N), T = N / 128;
  char* ptr = static_cast<char*>(scratch);
  const Bf16Workspace ws = bf16_workspace_carve(ptr, BH, S, CH);
  ptr += up256(bf16_workspace_bytes(BH, S, CH));
  const size_t rows = (size_t)BH * L, bhs = (size_t)BH * S;
  auto take = [&](size_t bytes) {
    char* r = ptr;
    ptr += up256(bytes);
    return r;
  };
  float* lse2 = reinterpret_cast<float*>(take(rows * 4));
  float* dpr = reinterpret_cast<float*>(take(rows * 4));
  float* GMp = reinterpret_cast<float*>(take(bhs * T * D * D * 4));
  float* Gzp = reinterpret_cast<float*>(take(bhs * T * D * 4));
  __nv_bfloat16* dMs = reinterpret_cast<__nv_bfloat16*>(take(bhs * 2 * D * D * 2));
  float* dzs = reinterpret_cast<float*>(take(bhs * D * 4));
  float* gzk = reinterpret_cast<float*>(take(bhs * T * D * 4));
  float* mem_part = reinterpret_cast<float*>(take(bhs * T * 4));
  float* dot_part = reinterpret_cast<float*>(take(bhs * T * 4));

  // M_{s-1} (bf16 hi/lo), z_{s-1} and, for Delta, every segment's G_s
  cudaError_t e = bf16_state_launch(k, v, M_in, z_in, nullptr, nullptr, ws, BH, L, N, S, CH, CL,
                                    mode, 0, stream);
  if (e != cudaSuccess) return e;

  const Bf16Layout lay = Bf16Layout::bhld(B, H, L);
  CUtensorMap mq, mk, mv, mdo, mm, mx, mg;
  if (!make_bf16_map4(&mq, q, (uint64_t)L, H, B, lay.q_sl, lay.q_sh, lay.q_sb, 128) ||
      !make_bf16_map4(&mk, k, (uint64_t)L, H, B, lay.q_sl, lay.q_sh, lay.q_sb, 128) ||
      !make_bf16_map4(&mv, v, (uint64_t)L, H, B, lay.q_sl, lay.q_sh, lay.q_sb, 128) ||
      !make_bf16_map4(&mdo, dout, (uint64_t)L, H, B, lay.q_sl, lay.q_sh, lay.q_sb, 128) ||
      !make_bf16_map(&mm, ws.Mhl, D, (uint64_t)bhs * 2, 128) ||
      !make_bf16_map(&mx, dMs, D, (uint64_t)bhs * 2, 128))
    return cudaErrorInvalidValue;
  if (mode == 1) {
    // G planes of the state path's dpart, fp32 [planes][128][128]; box 32 x 128
    EncodeTiledFn enc = get_encode_fn();
    const cuuint64_t dims[3] = {128, 128, (cuuint64_t)bhs * CH * 2};
    const cuuint64_t strides[2] = {128 * 4, 128 * 128 * 4};
    const cuuint32_t box[3] = {32, 128, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (!enc || enc(&mg, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ws.dpart, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    memset(&mg, 0, sizeof(mg));
  }
  BwdParams p;
  p.L = L;
  p.N = N;
  p.S = S;
  p.T = T;
  p.H = H;
  const long long tiles = (long long)BH * S * T;
  if (tiles >= (1ll << 31) || bhs >= (1ull << 31)) return cudaErrorInvalidValue;
  p.tiles = (unsigned)tiles;
  p.divT = FastDiv((uint32_t)T);
  p.divS = FastDiv((uint32_t)S);
  p.rsd = 0.08838834764831845f;
  p.sl = 1.4426950408889634f * p.rsd;

  mark(0);
  dq_bwd_kernel<<<p.tiles, kPipeThreads, kDqSmem, stream>>>(
      mq, mk, mv, mdo, mm, beta, ws.zprev, lse2, dpr, dot_part, mem_part, GMp, Gzp, dq, p);
  mark(1);
  chain_bwd_kernel<<<dim3(BH, 4), kChainThreads, kChainSmem, stream>>>(mg, GMp, dM_out, dM_in, dMs,
                                                                        S, CH, T, mode);
  if (mode == 0) dz_bwd_kernel<<<BH, D, 0, stream>>>(Gzp, gzk, dz_out, dzs, dz_in, S, T, mode);
  dkdv_bwd_kernel<<<p.tiles, kPipeThreads, kDkdvSmem, stream>>>(
      mq, mk, mv, mdo, mm, mx, beta, ws.zprev, lse2, dpr, dzs, gzk, dk, dv, p, mode);
  mark(2);
  if (mode == 1) {
    dz_bwd_kernel<<<BH, D, 0, stream>>>(Gzp, gzk, dz_out, dzs, dz_in, S, T, mode);
    const long long units = (long long)rows * (D / 8);
    const unsigned grid = (unsigned)min((units + 255) / 256, 148LL * 16);
    dk_dz_kernel<<<grid, 256, 0, stream>>>(k, dzs, dk, L, N, S, units);
  }
  dbeta_bwd_kernel<<<(H + 3) / 4, 128, 0, stream>>>(beta, mem_part, dot_part, dbeta, B, H, S, T);
  return cudaGetLastError();
}

}  // namespace infini
