// bf16_state.cu — compressive-memory state path of the bf16 forward (d = 128).
//
// The Linear+Delta rule of "Leave No Context Behind" (arXiv 2404.07143, as quoted
// on llm-papers-study.pages.dev, section 3.4),
//   M_s = M_{s-1} + sigma(K)^T (V - sigma(K) M_{s-1} / (sigma(K) z_{s-1})),
// is linear in M_{s-1} once z_{s-1} is known, and z does not depend on M (it is
// tracked the same way in both modes). With den_t = sigma(K_t) . z_{s-1} and
// inv_t = 1/den_t (0 when den_t == 0, i.e. the delta term is dropped),
//   M_s = M_{s-1} + dM_s - G_s M_{s-1},
//   dM_s = sigma(K_s)^T V_s,   G_s = sigma(K_s)^T diag(inv) sigma(K_s)   (d x d, symmetric).
// dM_s and G_s depend only on the segment's own tokens and z_{s-1}, so they are
// computed for every segment in parallel on the tensor cores; the sequential
// part shrinks to a d x d x d product per segment. The Linear rule is the same
// with G_s = 0. This is the same function as the per-token formula, evaluated in
// a different association order.
//
// Kernels (launch order):
//   zpart_kernel  : partial sums of sigma(K) per (head, segment, token chunk)
//   zscan_kernel  : z_{s-1} for every segment (fixed order), z_out
//   state_kernel  : bf16 tcgen05 GEMMs per (head, segment, chunk):
//                   [dM | G] = sigma(K)^T [V | diag(inv) sigma(K)]
//   chain_kernel  : per (head, 32-column block of M): M_{s-1} for every segment
//                   (written as a bf16 hi/lo pair for the retrieval GEMM), M_out.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "bf16_path.h"
#include "sm100.cuh"
#include "tma_map.h"

namespace infini {
namespace {

constexpr int D = 128;

__device__ __forceinline__ void bf16x8_to_f32(const uint4& raw, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// ---------------------------------------------------------------------------
// zpart: grid = BH * S * CH, block 256. zpart[idx][0..127] = sum over the chunk's
// tokens of sigma(K_t).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) zpart_kernel(const __nv_bfloat16* __restrict__ k,
                                                    float* __restrict__ zpart, long long L, int N,
                                                    int S, int CH, int CL) {
  __shared__ float red[16][D + 4];
  const long long idx = blockIdx.x;
  const int c = (int)(idx % CH);
  const int s = (int)((idx / CH) % S);
  const long long bh = idx / ((long long)CH * S);
  const long long t0 = (long long)s * N;
  const int n = (int)min((long long)N, L - t0);
  const int beg = min(n, c * CL), end = min(n, (c + 1) * CL);
  const int tid = threadIdx.x, cg = tid & 15, rg = tid >> 4;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  const __nv_bfloat16* base = k + ((size_t)bh * L + t0) * D + cg * 8;
  for (int t = beg + rg; t < end; t += 16) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(base + (size_t)t * D));
    float f[8];
    bf16x8_to_f32(raw, f);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += elu1(f[e]);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[rg][cg * 8 + e] = acc[e];
  __syncthreads();
  if (tid < D) {
    float sum = 0.f;
#pragma unroll
    for (int r = 0; r < 16; ++r) sum += red[r][tid];
    zpart[idx * D + tid] = sum;
  }
}

// ---------------------------------------------------------------------------
// zscan: grid = BH, block 128. zprev[bh][s] = z_in + sum_{r<s} dz_r; z_out = final.
// The thread that reads z_in[k] is the one that writes z_out[k] (in-place safe).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(D) zscan_kernel(const float* __restrict__ zpart,
                                                  const float* z_in, float* z_out,
                                                  float* __restrict__ zprev, int S, int CH) {
  const int bh = blockIdx.x, kf = threadIdx.x;
  float z = z_in ? z_in[(size_t)bh * D + kf] : 0.f;
  for (int s = 0; s < S; ++s) {
    zprev[((size_t)bh * S + s) * D + kf] = z;
    const float* zp = zpart + ((size_t)bh * S + s) * CH * D + kf;
    for (int c = 0; c < CH; ++c) z += zp[(size_t)c * D];
  }
  if (z_out) z_out[(size_t)bh * D + kf] = z;
}

// ---------------------------------------------------------------------------
// state_kernel: grid = BH * S * CH, one CTA per (head, segment, chunk of tokens).
//
// For the chunk's tokens it accumulates, in tensor memory,
//   columns   0..127: dM = sigma(K)^T V
//   columns 128..255: G  = sigma(K)^T diag(inv) sigma(K)      (Delta only)
// with bf16 tcgen05 MMAs (fp32 accumulation). sigma(K) is split into
// hi = rn_bf16(sigma) and lo = rn_bf16(sigma - hi), and dM = hi^T V + lo^T V
// (V is exact in bf16), which keeps dM within ~2^-16 relative per term. G sums
// only positive terms, so its bf16 rounding errors average out: G = hi^T (inv sigma)_bf16.
//
// Tokens move in slabs of 64. Per slab and pipeline stage (64 KB):
//   KH  [64 x 128] bf16: K as loaded by TMA, overwritten in place by sigma(K)_hi
//   V   [64 x 128] bf16: loaded by TMA, used as is
//   GH  [64 x 128] bf16: (inv * sigma(K))_bf16            (Delta only)
//   KL  [64 x 128] bf16: sigma(K)_lo
// each as two boxes of 64 features (8 KB), 128-byte swizzle, rows = tokens. As
// MMA operands they are MN-major (features contiguous, tokens = K); V and GH are
// adjacent so that hi^T [V | GH] is one N = 256 MMA.
// Warps 0..7 convert; warp 8 issues the TMA copies and the MMAs.
// ---------------------------------------------------------------------------
constexpr int kSlab = 64;
constexpr int kStages = 3;
constexpr int kBox = kSlab * 128;          // one 64-row x 64-feature box: 8 KB
constexpr int kMat = 2 * kBox;             // one [64 x 128] bf16 matrix: 16 KB
constexpr int OFF_KH = 0, OFF_V = kMat, OFF_GH = 2 * kMat, OFF_KL = 3 * kMat;
constexpr int kStageBytes = 4 * kMat;      // 64 KB
constexpr int kStateThreads = 288;
constexpr int kStateSmem = kStages * kStageBytes + 1024 + 1024;  // + alignment, barriers, z

__device__ __forceinline__ uint64_t slab_desc(uint32_t base, int kk) {
  // MN-major: 16 token rows per k-step (2048 B), 64-feature boxes kBox apart
  return sdesc(base + (uint32_t)kk * 2048, kBox, 1024);
}

__global__ void __launch_bounds__(kStateThreads, 1)
state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
             const float* __restrict__ zprev, float* __restrict__ dpart, long long L, int N, int S,
             int CH, int CL, int mode) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* bar_full = bars;                 // [kStages] TMA landed
  uint64_t* bar_conv = bars + kStages;       // [kStages] operands converted (256 arrivals)
  uint64_t* bar_mma = bars + 2 * kStages;    // [kStages] MMAs of the stage done
  uint64_t* bar_done = bars + 3 * kStages;   // all MMAs done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * kStages + 1);
  float* sZ = reinterpret_cast<float*>(smem + kStages * kStageBytes + 512);  // [128]

  const long long idx = blockIdx.x;
  const int c = (int)(idx % CH);
  const int s = (int)((idx / CH) % S);
  const long long bh = idx / ((long long)CH * S);
  const long long t0 = (long long)s * N;
  const int n = (int)min((long long)N, L - t0);
  const int beg = min(n, c * CL), end = min(n, (c + 1) * CL);
  const int len = end - beg;
  const int nslab = len > 0 ? (len + kSlab - 1) / kSlab : 0;
  const bool delta = mode == 1;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t ncols = delta ? 256u : 128u;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_conv[i], 256);
      mbar_init(&bar_mma[i], 1);
    }
    mbar_init(bar_done, 1);
    fence_barrier_init();
  }
  if (tid < D) sZ[tid] = delta ? zprev[((size_t)bh * S + s) * D + tid] : 0.f;
  if (warp == 8) {
    tmem_alloc(tmem_slot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  bool ok = true;

  if (warp == 8) {
    // ---------------- producer + MMA issuer ----------------
    if (lane == 0 && nslab > 0) {
      const int row0 = (int)(t0 + beg);
      auto load = [&](int sl) {
        uint8_t* st = smem + (sl % kStages) * kStageBytes;
        uint64_t* fb = &bar_full[sl % kStages];
        mbar_arrive_expect_tx(fb, 2 * kMat);
        const int row = row0 + sl * kSlab;
        tma_load_3d(st + OFF_KH, &tm_k, fb, 0, row, (int)bh);
        tma_load_3d(st + OFF_KH + kBox, &tm_k, fb, 64, row, (int)bh);
        tma_load_3d(st + OFF_V, &tm_v, fb, 0, row, (int)bh);
        tma_load_3d(st + OFF_V + kBox, &tm_v, fb, 64, row, (int)bh);
      };
      int issued = 0;
      for (; issued < nslab && issued < kStages; ++issued) load(issued);
      const uint32_t id256 = idesc_f32acc(1, 1, 1, 128, 256);
      const uint32_t id128 = idesc_f32acc(1, 1, 1, 128, 128);
      for (int sl = 0; sl < nslab && ok; ++sl) {
        const int stg = sl % kStages;
        if (!mbar_wait(&bar_conv[stg], (uint32_t)((sl / kStages) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t base = smem_u32(smem + stg * kStageBytes);
#pragma unroll
        for (int kk = 0; kk < kSlab / 16; ++kk) {
          const uint32_t acc = (sl > 0 || kk > 0) ? 1u : 0u;
          const uint64_t a_hi = slab_desc(base + OFF_KH, kk);
          const uint64_t a_lo = slab_desc(base + OFF_KL, kk);
          const uint64_t b_v = slab_desc(base + OFF_V, kk);
          if (delta) {
            mma_bf16_ss(tmem_d, a_hi, b_v, id256, acc);  // [dM | G] += hi^T [V | GH]
          } else {
            mma_bf16_ss(tmem_d, a_hi, b_v, id128, acc);  // dM += hi^T V
          }
          mma_bf16_ss(tmem_d, a_lo, b_v, id128, 1u);     // dM += lo^T V
        }
        mma_commit(&bar_mma[stg]);
        // refill the stage used by slab sl - 1 once its MMAs are done
        if (sl >= 1 && issued < nslab) {
          const int prev = sl - 1;
          if (!mbar_wait(&bar_mma[prev % kStages], (uint32_t)((prev / kStages) & 1))) {
            ok = false;
            break;
          }
          load(issued++);
        }
      }
      mma_commit(bar_done);
    } else if (lane == 0) {
      mma_commit(bar_done);  // nothing issued: completes at once
    }
  } else {
    // ---------------- converters (warps 0..7) ----------------
    for (int sl = 0; sl < nslab && ok; ++sl) {
      const int stg = sl % kStages;
      uint8_t* st = smem + stg * kStageBytes;
      if (!mbar_wait(&bar_full[stg], (uint32_t)((sl / kStages) & 1))) {
        ok = false;
        break;
      }
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int item = tid + 256 * it;
        const int r = item >> 4, cg = item & 15;  // token row in the slab, 8-feature group
        const bool valid = sl * kSlab + r < len;
        const uint32_t off = (uint32_t)(cg >> 3) * kBox + sw128(r, cg & 7);
        const uint4 raw = *reinterpret_cast<const uint4*>(st + OFF_KH + off);
        float f[8];
        bf16x8_to_f32(raw, f);
        float den = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          f[e] = valid ? elu1(f[e]) : 0.f;
          den = fmaf(f[e], sZ[cg * 8 + e], den);
        }
        // 16 lanes of a half-warp hold the 128 features of one token
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
        uint32_t hi[4], lo[4], gh[4];
        const float inv = (delta && den != 0.f) ? 1.f / den : 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
          const float2 hf = __bfloat1622float2(h);
          const __nv_bfloat162 l = __floats2bfloat162_rn(f[2 * e] - hf.x, f[2 * e + 1] - hf.y);
          const __nv_bfloat162 g = __floats2bfloat162_rn(f[2 * e] * inv, f[2 * e + 1] * inv);
          hi[e] = *reinterpret_cast<const uint32_t*>(&h);
          lo[e] = *reinterpret_cast<const uint32_t*>(&l);
          gh[e] = *reinterpret_cast<const uint32_t*>(&g);
        }
        *reinterpret_cast<uint4*>(st + OFF_KH + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(st + OFF_KL + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        if (delta)
          *reinterpret_cast<uint4*>(st + OFF_GH + off) = make_uint4(gh[0], gh[1], gh[2], gh[3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&bar_conv[stg]);
    }
  }

  const bool done = mbar_wait(bar_done, 0);
  tc_fence_after();
  // epilogue: warps 0-3 write dM rows, warps 4-7 write G rows (Delta)
  if (warp < 8) {
    const int lane_base = (warp & 3) * 32;
    const int row = lane_base + lane;
    const int half = warp >> 2;
    if (half == 0 || delta) {
      float* dst = dpart + ((size_t)idx * 2 + half) * D * D + (size_t)row * D;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t rr[32];
        if (nslab > 0) {
          tmem_ld32(tmem_d + ((uint32_t)lane_base << 16) + half * 128 + cc * 32, rr);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) rr[e] = 0u;
        }
        if (done && ok) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + cc * 32 + e) =
                make_float4(__uint_as_float(rr[e]), __uint_as_float(rr[e + 1]),
                            __uint_as_float(rr[e + 2]), __uint_as_float(rr[e + 3]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem_d, ncols);
  }
}

// ---------------------------------------------------------------------------
// chain_kernel: grid = (BH, 4), block 256. Column block cb covers M[:, 32cb .. 32cb+31].
// Thread t owns a 4x4 tile: rows 4*(t/8) .. +3, columns 32cb + 4*(t%8) .. +3.
// For s = 0..S-1: write M_{s-1} as hi/lo bf16 into Mhl[bh][s] (hi = rn(M),
// lo = rn(M - hi)), then M += dM_s - G_s M (Delta) or M += dM_s (Linear).
// G_s is symmetric, so row k of G_s serves as column k.
// ---------------------------------------------------------------------------
constexpr int kChainSmem = (D * D + D * 32) * 4;

__global__ void __launch_bounds__(256, 1)
chain_kernel(const float* __restrict__ dpart, const float* M_in, float* M_out,
             __nv_bfloat16* __restrict__ Mhl, int S, int CH, int mode) {
  extern __shared__ __align__(16) float csm[];
  float* sG = csm;            // [128][128]
  float* sM = csm + D * D;    // [128][32]
  const int bh = blockIdx.x, cb = blockIdx.y, tid = threadIdx.x;
  const int r0 = 4 * (tid >> 3), cl = 4 * (tid & 7), c0 = 32 * cb + cl;
  const bool delta = mode == 1;
  float m[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float4 t = M_in ? *reinterpret_cast<const float4*>(M_in + ((size_t)bh * D + r0 + i) * D + c0)
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    m[i][0] = t.x; m[i][1] = t.y; m[i][2] = t.z; m[i][3] = t.w;
  }
  for (int s = 0; s < S; ++s) {
    __nv_bfloat16* hi = Mhl + ((size_t)bh * S + s) * 2 * D * D;
    __nv_bfloat16* lo = hi + D * D;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h01 = __floats2bfloat162_rn(m[i][0], m[i][1]);
      __nv_bfloat162 h23 = __floats2bfloat162_rn(m[i][2], m[i][3]);
      const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
      __nv_bfloat162 l01 = __floats2bfloat162_rn(m[i][0] - f01.x, m[i][1] - f01.y);
      __nv_bfloat162 l23 = __floats2bfloat162_rn(m[i][2] - f23.x, m[i][3] - f23.y);
      uint2 hv, lv;
      hv.x = *reinterpret_cast<uint32_t*>(&h01); hv.y = *reinterpret_cast<uint32_t*>(&h23);
      lv.x = *reinterpret_cast<uint32_t*>(&l01); lv.y = *reinterpret_cast<uint32_t*>(&l23);
      *reinterpret_cast<uint2*>(hi + (size_t)(r0 + i) * D + c0) = hv;
      *reinterpret_cast<uint2*>(lo + (size_t)(r0 + i) * D + c0) = lv;
    }
    float dm[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) dm[i][j] = 0.f;
    const float* dp = dpart + ((size_t)bh * S + s) * CH * 2 * D * D;
    for (int c = 0; c < CH; ++c) {
      const float* p = dp + (size_t)c * 2 * D * D;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 t = *reinterpret_cast<const float4*>(p + (size_t)(r0 + i) * D + c0);
        dm[i][0] += t.x; dm[i][1] += t.y; dm[i][2] += t.z; dm[i][3] += t.w;
      }
    }
    if (delta) {
      __syncthreads();  // previous iteration's readers of sG / sM are done
      for (int e = tid * 4; e < D * D; e += 256 * 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int c = 0; c < CH; ++c) {
          const float4 t = *reinterpret_cast<const float4*>(dp + (size_t)c * 2 * D * D + D * D + e);
          acc.x += t.x; acc.y += t.y; acc.z += t.z; acc.w += t.w;
        }
        *reinterpret_cast<float4*>(sG + e) = acc;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
        *reinterpret_cast<float4*>(sM + (r0 + i) * 32 + cl) =
            make_float4(m[i][0], m[i][1], m[i][2], m[i][3]);
      __syncthreads();
      float gm[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) gm[i][j] = 0.f;
#pragma unroll 4
      for (int kk = 0; kk < D; ++kk) {
        const float4 g4 = *reinterpret_cast<const float4*>(sG + kk * D + r0);   // G[r0..r0+3][kk]
        const float4 m4 = *reinterpret_cast<const float4*>(sM + kk * 32 + cl);  // M[kk][c..c+3]
        const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
        const float mv[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) gm[i][j] = fmaf(gv[i], mv[j], gm[i][j]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) m[i][j] += dm[i][j] - gm[i][j];
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) m[i][j] += dm[i][j];
    }
  }
  if (M_out) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<float4*>(M_out + ((size_t)bh * D + r0 + i) * D + c0) =
          make_float4(m[i][0], m[i][1], m[i][2], m[i][3]);
  }
}

}  // namespace

void bf16_state_plan(int BH, int S, int N, int* CH, int* CL) {
  // Chunk the segments so that the state GEMM has at least ~2 CTAs per SM, with
  // chunks of at least 128 tokens.
  const long long units = (long long)BH * S;
  int ch = 1;
  const int maxch = N >= 128 ? N / 128 : 1;
  while (units * ch < 296 && ch * 2 <= maxch) ch *= 2;
  *CH = ch;
  *CL = (N + ch - 1) / ch;
}

cudaError_t bf16_state_set_attributes() {
  cudaError_t e =
      cudaFuncSetAttribute(state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kStateSmem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kChainSmem);
}

size_t bf16_workspace_bytes(int BH, int S, int CH) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t bhs = (size_t)BH * S;
  return up(bhs * CH * D * 4) + up(bhs * D * 4) + up(bhs * CH * 2 * D * D * 4) +
         up(bhs * 2 * D * D * 2);
}

Bf16Workspace bf16_workspace_carve(void* base, int BH, int S, int CH) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t bhs = (size_t)BH * S;
  char* p = static_cast<char*>(base);
  Bf16Workspace w;
  w.zpart = reinterpret_cast<float*>(p);
  p += up(bhs * CH * D * 4);
  w.zprev = reinterpret_cast<float*>(p);
  p += up(bhs * D * 4);
  w.dpart = reinterpret_cast<float*>(p);
  p += up(bhs * CH * 2 * D * D * 4);
  w.Mhl = reinterpret_cast<__nv_bfloat16*>(p);
  return w;
}

cudaError_t bf16_state_launch(const __nv_bfloat16* k, const __nv_bfloat16* v, const float* M_in,
                              const float* z_in, float* M_out, float* z_out,
                              const Bf16Workspace& ws, int BH, long long L, int N, int S, int CH,
                              int CL, int mode, cudaStream_t stream) {
  const unsigned nunits = (unsigned)((long long)BH * S * CH);
  zpart_kernel<<<nunits, 256, 0, stream>>>(k, ws.zpart, L, N, S, CH, CL);
  zscan_kernel<<<BH, D, 0, stream>>>(ws.zpart, z_in, z_out, ws.zprev, S, CH);
  CUtensorMap mk, mv;
  if (!make_bf16_map(&mk, k, (uint64_t)L, BH, kSlab) || !make_bf16_map(&mv, v, (uint64_t)L, BH, kSlab))
    return cudaErrorInvalidValue;
  state_kernel<<<nunits, kStateThreads, kStateSmem, stream>>>(mk, mv, ws.zprev, ws.dpart, L, N, S,
                                                               CH, CL, mode);
  chain_kernel<<<dim3(BH, 4), 256, mode == 1 ? kChainSmem : 0, stream>>>(ws.dpart, M_in, M_out,
                                                                        ws.Mhl, S, CH, mode);
  return cudaGetLastError();
}

}  // namespace infini
