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
// Kernels (launch order; Linear+Delta: zpart, zscan, state, chain;
// Linear: state (which also sums sigma(K)), zscan, chain):
//   zpart_kernel  : partial sums of sigma(K) per (head, segment, token chunk)
//   zscan_kernel  : z_{s-1} for every segment (fixed order), z_out
//   state_kernel  : bf16 tcgen05 GEMMs per (head, segment, chunk):
//                   [dM | G] = sigma(K)^T [V | diag(inv) sigma(K)]
//   chain_kernel  : per (head, 32-column block of M): M_{s-1} for every segment
//                   (written as a bf16 hi/lo pair for the retrieval GEMM), M_out.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <cstring>

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
                                                    int S, int CH, int CL, int Hkv, long long sb,
                                                    long long sh, long long sl) {
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
  // key/value head bh = (batch row, head); rows of K are sl elements apart
  const __nv_bfloat16* base = k + (bh / Hkv) * sb + (bh % Hkv) * sh + t0 * sl + cg * 8;
  // four rows per thread in flight: one outstanding load per thread would cap the
  // stream at ~4 TB/s
  int t = beg + rg;
  for (; t + 48 < end; t += 64) {
    uint4 raw[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      raw[u] = __ldg(reinterpret_cast<const uint4*>(base + (t + 16 * u) * sl));
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float f[8];
      bf16x8_to_f32(raw[u], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += elu1(f[e]);
    }
  }
  for (; t < end; t += 16) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(base + t * sl));
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
// In Linear mode the chain kernel runs the same scan in its otherwise idle warp.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void zscan_feature(const float* __restrict__ zpart, const float* z_in,
                                              float* z_out, float* __restrict__ zprev, int S,
                                              int CH, int first, int bh, int kf) {
  float z = z_in ? z_in[(size_t)bh * D + kf] : 0.f;
  const float* zp = zpart + (size_t)bh * S * CH * D + kf;
  if (CH == 1) {
    // four segments' sums loaded together (their loads do not wait on z); still added
    // in segment order
    int s = 0;
    for (; s + 4 <= S; s += 4) {
      float t[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) t[e] = __ldcg(zp + (size_t)(s + e) * D);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (s + e >= first) zprev[((size_t)bh * S + s + e) * D + kf] = z;
        z += t[e];
      }
    }
    for (; s < S; ++s) {
      if (s >= first) zprev[((size_t)bh * S + s) * D + kf] = z;
      z += __ldcg(zp + (size_t)s * D);
    }
  } else {
    for (int s = 0; s < S; ++s) {
      if (s >= first) zprev[((size_t)bh * S + s) * D + kf] = z;
      for (int c = 0; c < CH; ++c) z += __ldcg(zp + ((size_t)s * CH + c) * D);
    }
  }
  if (z_out) z_out[(size_t)bh * D + kf] = z;
}

__global__ void __launch_bounds__(D) zscan_kernel(const float* __restrict__ zpart,
                                                  const float* z_in, float* z_out,
                                                  float* __restrict__ zprev, int S, int CH,
                                                  int first) {
  zscan_feature(zpart, z_in, z_out, zprev, S, CH, first, blockIdx.x, threadIdx.x);
}

// ---------------------------------------------------------------------------
// state_kernel: persistent, min(BH * S * CH, SMs) CTAs; each walks the units (head,
// segment, chunk of tokens) blockIdx.x, blockIdx.x + gridDim.x, ... with its ring and
// barrier phases running on from one unit to the next, so the next unit's copies
// stream while the converter warps drain the last unit's sums.
//
// For a unit's tokens it accumulates, in tensor memory,
//   columns   0..127: dM = sigma(K)^T V
//   columns 128..255: G  = sigma(K)^T diag(inv) sigma(K)      (Delta only)
// with bf16 tcgen05 MMAs (fp32 accumulation). sigma(K) is split into
// hi = rn_bf16(sigma) and lo = rn_bf16(sigma - hi), and dM = hi^T V + lo^T V
// (V is exact in bf16), which keeps dM within ~2^-16 relative per term. G sums
// only positive terms, so its bf16 rounding errors average out: G = hi^T (inv sigma)_bf16.
// In Linear mode the kernel also writes the chunk's sum of sigma(K) (zpart), so
// K is read once.
//
// Tokens move in slabs of 64 through a ring of 3 stages. Per stage (64 KB):
//   KH  [64 x 128] bf16: K as loaded by TMA, overwritten in place by sigma(K)_hi
//   V   [64 x 128] bf16: loaded by TMA, used as is
//   GH  [64 x 128] bf16: (inv * sigma(K))_bf16            (Delta only)
//   KL  [64 x 128] bf16: sigma(K)_lo
// each as two boxes of 64 features (4 KB), 128-byte swizzle, rows = tokens. As
// MMA operands they are MN-major (features contiguous, tokens = K); V and GH are
// adjacent so that hi^T [V | GH] is one N = 256 MMA.
// Warps 0..15 convert (one 8-feature group of two tokens each per slab: 64-token
// slabs measured ~6% faster for this kernel than 32-token ones with twice the
// stages, the per-slab waits and arrivals being paid on twice the work) and drain
// each unit's sums, warp 16 issues the TMA copies, warp 17 issues the MMAs.
// ---------------------------------------------------------------------------
constexpr int kSlab = 64;
constexpr int kStages = 3;
constexpr int kConvRows = 32;  // token rows converted at once (16 threads per row)
constexpr int kBox = kSlab * 128;          // one 64-row x 64-feature box: 8 KB
constexpr int kMat = 2 * kBox;             // one [64 x 128] bf16 matrix: 16 KB
constexpr int OFF_KH = 0, OFF_V = kMat, OFF_GH = 2 * kMat, OFF_KL = 3 * kMat;
constexpr int kStageBytes = 4 * kMat;      // 64 KB
constexpr int kConvWarps = 16;
constexpr int kStateThreads = (kConvWarps + 2) * 32;
constexpr int kProdWarp = kConvWarps, kMmaWarp = kConvWarps + 1;
constexpr int kZredBytes = kConvRows * 128 * 4;   // 16 KB
constexpr int kStateSmem = kStages * kStageBytes + kZredBytes + 1024 + 256;  // + alignment, barriers

__device__ __forceinline__ uint32_t tf32_rna(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// Bounded wait used only while draining after an error: ignores the error flag.
__device__ __forceinline__ void drain_wait_s(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) break;  // 200 ms
  }
}

__device__ __forceinline__ uint64_t slab_desc(uint32_t base, int kk) {
  // MN-major: 16 token rows per k-step (2048 B), 64-feature boxes kBox apart
  return sdesc(base + (uint32_t)kk * 2048, kBox, 1024);
}

__global__ void __launch_bounds__(kStateThreads, 1)
state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
             const float* __restrict__ zprev, float* __restrict__ dpart,
             float* __restrict__ zpart, long long L, int N, int S, int CH, int CL, int mode,
             int zsum, int Hkv, long long nunits) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  // [32][128] partial sums of sigma(K) of one unit (its own area: the ring keeps
  // streaming the next unit meanwhile)
  float* sZred = reinterpret_cast<float*>(smem + kStages * kStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes + kZredBytes);
  uint64_t* bar_full = bars;                 // [kStages] TMA landed
  uint64_t* bar_conv = bars + kStages;       // [kStages] operands converted (warp arrivals)
  uint64_t* bar_mma = bars + 2 * kStages;    // [kStages] MMAs of the stage done
  uint64_t* bar_done = bars + 3 * kStages;   // a unit's MMAs all done (once per unit)
  uint64_t* bar_drain = bars + 3 * kStages + 1;  // every MMA of the CTA done (at the end)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * kStages + 2);

  const bool delta = mode == 1;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t ncols = delta ? 256u : 128u;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_conv[i], kConvWarps);  // one arrival per converter warp
      mbar_init(&bar_mma[i], 1);
    }
    mbar_init(bar_done, 1);
    mbar_init(bar_drain, 1);
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  bool ok = true;
  const int cg = tid & 15;  // this converter's 8-feature group
  const int r = tid >> 4;   // this converter's token row in each slab

  // unit idx = (head, segment, token chunk): its head, first row, tokens and slabs
  struct Unit {
    long long bh, row0;
    int s, len, nslab;
  };
  auto unit = [&](long long idx) {
    Unit x;
    const int c = (int)(idx % CH);
    x.s = (int)((idx / CH) % S);
    x.bh = idx / ((long long)CH * S);
    const long long t0 = (long long)x.s * N;
    const int n = (int)min((long long)N, L - t0);
    const int beg = min(n, c * CL), end = min(n, (c + 1) * CL);
    x.len = end - beg;
    x.nslab = x.len > 0 ? (x.len + kSlab - 1) / kSlab : 0;
    x.row0 = t0 + beg;
    return x;
  };

  if (warp == kProdWarp) {
    // ---------------- TMA producer: the ring runs on across units ----------------
    if (lane == 0) {
      int g = 0;
      int issued[kStages] = {0, 0, 0};
      for (long long idx = blockIdx.x; ok && idx < nunits; idx += gridDim.x) {
        const Unit x = unit(idx);
        const int hh = (int)(x.bh % Hkv), bb = (int)(x.bh / Hkv);
        for (int sl = 0; sl < x.nslab; ++sl, ++g) {
          const int stg = g % kStages;
          if (g >= kStages && !mbar_wait(&bar_mma[stg], (uint32_t)((g / kStages - 1) & 1))) {
            ok = false;
            break;
          }
          uint8_t* st = smem + stg * kStageBytes;
          mbar_arrive_expect_tx(&bar_full[stg], 2 * kMat);
          const int row = (int)(x.row0 + sl * kSlab);
          tma_load_4d(st + OFF_KH, &tm_k, &bar_full[stg], 0, row, hh, bb);
          tma_load_4d(st + OFF_KH + kBox, &tm_k, &bar_full[stg], 64, row, hh, bb);
          tma_load_4d(st + OFF_V, &tm_v, &bar_full[stg], 0, row, hh, bb);
          tma_load_4d(st + OFF_V + kBox, &tm_v, &bar_full[stg], 64, row, hh, bb);
          ++issued[stg];
        }
      }
      if (!ok)  // let the copies already issued land before the CTA exits
        for (int st = 0; st < kStages; ++st)
          if (issued[st] > 0) drain_wait_s(&bar_full[st], (uint32_t)((issued[st] - 1) & 1));
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer ----------------
    // The whole warp runs the loop and waits; one elected lane (always lane 0)
    // issues and commits, which keeps the issue path short next to the busy
    // converter warps on the same scheduler. A unit's first product overwrites the
    // accumulator: the converters read the previous unit's sums out of it before
    // they convert (and signal) the first slab of this one.
    const uint32_t id256 = idesc_f32acc(1, 1, 1, 128, 256);
    const uint32_t id128 = idesc_f32acc(1, 1, 1, 128, 128);
    int g = 0;
    for (long long idx = blockIdx.x; ok && idx < nunits; idx += gridDim.x) {
      const Unit x = unit(idx);
      for (int sl = 0; sl < x.nslab; ++sl, ++g) {
        const int stg = g % kStages;
        if (!mbar_wait_warp(&bar_conv[stg], (uint32_t)((g / kStages) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t base = smem_u32(smem + stg * kStageBytes);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kSlab / 16; ++kk) {
            const uint32_t acc = (sl > 0 || kk > 0) ? 1u : 0u;
            const uint64_t a_hi = slab_desc(base + OFF_KH, kk);
            const uint64_t a_lo = slab_desc(base + OFF_KL, kk);
            const uint64_t b_v = slab_desc(base + OFF_V, kk);
            mma_bf16_ss(tmem_d, a_hi, b_v, delta ? id256 : id128, acc);  // [dM | G] += hi^T [V | GH]
            mma_bf16_ss(tmem_d, a_lo, b_v, id128, 1u);                  // dM += lo^T V
          }
          mma_commit(&bar_mma[stg]);
        }
        __syncwarp();
      }
      // the unit's sums are complete (also after an error, so that the converters never
      // wait on a phase that cannot come). A unit without tokens has no products and
      // no commit: two commits with no converter wait between them would let the
      // barrier complete twice before its waiters saw the first.
      if (x.nslab > 0) {
        if (elect_one()) mma_commit(bar_done);
        __syncwarp();
      }
    }
    // no product may still be running when the CTA frees tensor memory (the converters
    // stop waiting for the units' sums after an error)
    if (elect_one()) mma_commit(bar_drain);
    __syncwarp();
    drain_wait_s(bar_drain, 0);
  } else {
    // ---------------- converters (warps 0..15), then each unit's epilogue ----------------
    int g = 0, un = 0;  // un: units with tokens so far (bar_done completes once for each)
    for (long long idx = blockIdx.x; idx < nunits; idx += gridDim.x) {
      const Unit x = unit(idx);
      float dz[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // sum of sigma(K)
      float zr[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        zr[e] = delta ? zprev[((size_t)x.bh * S + x.s) * D + cg * 8 + e] : 0.f;
      for (int sl = 0; sl < x.nslab && ok; ++sl, ++g) {
        const int stg = g % kStages;
        uint8_t* st = smem + stg * kStageBytes;
        if (!mbar_wait_warp(&bar_full[stg], (uint32_t)((g / kStages) & 1))) {
          ok = false;
          break;
        }
#pragma unroll
        for (int rh = 0; rh < kSlab / kConvRows; ++rh) {
          const int row = r + kConvRows * rh;
          const bool valid = sl * kSlab + row < x.len;
          const uint32_t off = (uint32_t)(cg >> 3) * kBox + sw128(row, cg & 7);
          const uint4 raw = *reinterpret_cast<const uint4*>(st + OFF_KH + off);
          float f[8];
          bf16x8_to_f32(raw, f);
          // sigma(K), every exponential on the MUFU: the converters are bound by their
          // instruction issue, and the FMA-pipe polynomial costs more instructions (with
          // half of the exponentials on it the state path was 3-4% slower, measured at
          // the 1B-layer shape in both modes)
          float den = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = elu1(f[e]);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            f[e] = valid ? f[e] : 0.f;
            den = fmaf(f[e], zr[e], den);
            dz[e] += f[e];
          }
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
            const float2 hf = __bfloat1622float2(h);
            const __nv_bfloat162 l = __floats2bfloat162_rn(f[2 * e] - hf.x, f[2 * e + 1] - hf.y);
            hi[e] = *reinterpret_cast<const uint32_t*>(&h);
            lo[e] = *reinterpret_cast<const uint32_t*>(&l);
          }
          *reinterpret_cast<uint4*>(st + OFF_KH + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(st + OFF_KL + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
          if (delta) {
            // 16 lanes of a half-warp hold the 128 features of one token
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
            const float inv = den != 0.f ? 1.f / den : 0.f;
            uint32_t gh[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 g2 = __floats2bfloat162_rn(f[2 * e] * inv, f[2 * e + 1] * inv);
              gh[e] = *reinterpret_cast<const uint32_t*>(&g2);
            }
            *reinterpret_cast<uint4*>(st + OFF_GH + off) = make_uint4(gh[0], gh[1], gh[2], gh[3]);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive_warp(&bar_conv[stg]);
      }
      if (!ok) break;
      if (x.nslab > 0) {
        if (!mbar_wait_warp(bar_done, (uint32_t)(un & 1))) {
          ok = false;
          break;
        }
        ++un;
        tc_fence_after();
      }
      // epilogue: every converter warp drains 32 rows (its tensor-memory lane quadrant)
      // x 32 columns of [dM | G]: column chunk (warp >> 2) of dM and, for Delta, the G
      // chunk four further on; each thread writes its row's 128 bytes as four 256-bit
      // stores (whole 32-byte sectors)
      const int lane_base = (warp & 3) * 32;
      const int row = lane_base + lane;
      for (int k = 0; k < (delta ? 2 : 1); ++k) {
        const int cc = (warp >> 2) + 4 * k;  // 0..3: dM columns, 4..7: G columns
        uint32_t rr[32];
        if (x.nslab > 0) {
          tmem_ld32(tmem_d + ((uint32_t)lane_base << 16) + (uint32_t)cc * 32, rr);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) rr[e] = 0u;
        }
        if (cc >= 4) {  // G feeds a tf32 MMA in the chain: round it here, unbiased
#pragma unroll
          for (int e = 0; e < 32; ++e) rr[e] = tf32_rna(__uint_as_float(rr[e]));
        }
        float* dst = dpart + ((size_t)idx * 2 + (cc >> 2)) * D * D + (size_t)row * D + (cc & 3) * 32;
#pragma unroll
        for (int e = 0; e < 32; e += 8) st_global_v8(dst + e, rr + e);
      }
      // the accumulator is read: the next unit's first product may overwrite it (the
      // MMA warp issues it only after this warp's arrival for that unit's first slab)
      tc_fence_before();
      if (zsum) {
        // unit sum of sigma(K): threads with the same feature group add up
#pragma unroll
        for (int e = 0; e < 8; ++e) sZred[r * 128 + cg * 8 + e] = dz[e];
        named_bar_sync(1, kConvWarps * 32);
        if (tid < D) {
          float sum = 0.f;
#pragma unroll
          for (int rr = 0; rr < kConvRows; ++rr) sum += sZred[rr * 128 + tid];
          zpart[idx * D + tid] = sum;
        }
        named_bar_sync(1, kConvWarps * 32);  // sZred is rewritten by the next unit
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_d, ncols);
  }
}

// ---------------------------------------------------------------------------
// chain_kernel: grid = (BH, 4), block 160. Column block cb covers M[:, 32cb .. 32cb+31].
// Threads 0..127 own one row r of the block (32 fp32 values in registers);
// warp 4 issues the TMA copies of G and the MMAs.
// For s = 0..S-1: write M_{s-1} as hi/lo bf16 into Mhl[bh][s] (hi = rn(M),
// lo = rn(M - hi)), then M += dM_s (Linear) or M += dM_s - G_s M (Delta).
// G_s M runs on the tensor cores as tf32 (both operands K-major): A = G_s as
// stored (row-major, rounded to tf32 by the state kernel), B = the block of M
// transposed in shared memory (rounded to tf32); D [128 x 32] in tensor memory.
// G_s of the next segment is prefetched by TMA while the current one is used.
// ---------------------------------------------------------------------------
constexpr int kChainThreads = 160;
constexpr int kGBytes = D * D * 4;                 // 64 KB
constexpr int kMtBytes = 32 * D * 4;               // 16 KB: M block transposed [32][128]
constexpr int kChainSmem = 2 * kGBytes + kMtBytes + 1024 + 256;

__global__ void __launch_bounds__(kChainThreads, 1)
chain_kernel(const __grid_constant__ CUtensorMap tm_g, const float* __restrict__ dpart,
             const float* M_in, float* M_out, __nv_bfloat16* __restrict__ Mhl, int S, int CH,
             int mode, int first, const float* __restrict__ zpart, const float* z_in,
             float* z_out, float* __restrict__ zprev) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sG = smem;                         // 2 buffers x [4 boxes of 128 rows x 32 fp32]
  uint8_t* sMt = smem + 2 * kGBytes;          // [4 boxes of 32 rows x 32 fp32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * kGBytes + kMtBytes);
  uint64_t* bar_g = bars;       // [2] G landed
  uint64_t* bar_mt = bars + 2;  // M^T written (4 warp arrivals)
  uint64_t* bar_mma = bars + 3; // one G_c M product done (per chunk; the MMA thread waits it)
  uint64_t* bar_seg = bars + 4; // G_s M of a whole segment done (once per segment)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 5);

  const int bh = blockIdx.x, cb = blockIdx.y, tid = threadIdx.x, warp = tid >> 5;
  const int c0 = 32 * cb;
  const bool delta = mode == 1;
  if (tid == 0) {
    mbar_init(&bar_g[0], 1);
    mbar_init(&bar_g[1], 1);
    mbar_init(bar_mt, 4);  // one arrival per row warp
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
    // Linear (zpart given): this warp scans z for features [32 cb, 32 cb + 32) of the
    // head, beside the rows' M chain (the two do not depend on each other).
    if (!delta && zpart)
      zscan_feature(zpart, z_in, z_out, zprev, S, CH, first, bh, c0 + (tid & 31));
    // The whole warp runs the loop and waits; one elected lane (always lane 0)
    // issues the copies, MMAs and commits.
    if (delta) {
      // G_s of chunk c: plane (bh*S + s)*CH*2 + 2c + 1 of dpart
      auto load_g = [&](int s, int c, int buf) {
        if (elect_one()) {
          mbar_arrive_expect_tx(&bar_g[buf], kGBytes);
          const int plane = ((bh * S + s) * CH + c) * 2 + 1;
#pragma unroll
          for (int bx = 0; bx < 4; ++bx)
            tma_load_3d(sG + buf * kGBytes + bx * (D * 128), &tm_g, &bar_g[buf], bx * 32, 0,
                        plane);
        }
        __syncwarp();
      };
      const uint32_t idesc = idesc_f32acc(2, 0, 0, 128, 32);
      int n = 0;  // G loads consumed so far
      const int total = S * CH;
      load_g(0, 0, 0);
      for (int s = 0; s < S && ok; ++s) {
        // M^T of this segment's M_{s-1} must be in shared memory
        if (!mbar_wait_warp(bar_mt, (uint32_t)(s & 1))) {
          ok = false;
          break;
        }
        for (int c = 0; c < CH; ++c, ++n) {
          const int buf = n & 1;
          if (n + 1 < total) {
            // the other buffer was last read by the MMA of load n-1, finished before
            // this point (its commit was awaited below)
            load_g((n + 1) / CH, (n + 1) % CH, buf ^ 1);
          }
          if (!mbar_wait_warp(&bar_g[buf], (uint32_t)((n >> 1) & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ga = smem_u32(sG + buf * kGBytes), mb = smem_u32(sMt);
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < D / 8; ++kk) {
              const uint32_t koff = (uint32_t)(kk >> 2) * (D * 128) + (uint32_t)(kk & 3) * 32;
              const uint32_t moff = (uint32_t)(kk >> 2) * (32 * 128) + (uint32_t)(kk & 3) * 32;
              mma_tf32_ss(tmem_d, sdesc(ga + koff, 16, 1024), sdesc(mb + moff, 16, 1024), idesc,
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
    }
  } else {
    const int r = tid;  // row of M
    float m[32];
    if (M_in) {
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const float4 t = *reinterpret_cast<const float4*>(M_in + ((size_t)bh * D + r) * D + c0 + e);
        m[e] = t.x; m[e + 1] = t.y; m[e + 2] = t.z; m[e + 3] = t.w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) m[e] = 0.f;
    }
    // dM of a later segment, prefetched into registers. Chunk 0 is loaded by plain
    // assignment so that nothing waits on the loads until the segment uses them;
    // further chunks (only when a segment is split, e.g. one-segment steps) are added
    // at once.
    auto load_dm = [&](float (&dst)[32], int s) {
      const float* src = dpart + ((size_t)((bh * S + s) * CH) * 2) * D * D + (size_t)r * D + c0;
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const float4 t = __ldg(reinterpret_cast<const float4*>(src + e));
        dst[e] = t.x; dst[e + 1] = t.y; dst[e + 2] = t.z; dst[e + 3] = t.w;
      }
      for (int c = 1; c < CH; ++c) {
        const float* sc = src + (size_t)c * 2 * D * D;
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 t = __ldg(reinterpret_cast<const float4*>(sc + e));
          dst[e] += t.x; dst[e + 1] += t.y; dst[e + 2] += t.z; dst[e + 3] += t.w;
        }
      }
    };
    // M_{s-1} -> hi / lo bf16 (segments below `first` were written by prep_first_kernel)
    auto emit = [&](int s) {
      if (s < first) return;
      __nv_bfloat16* hi = Mhl + ((size_t)bh * S + s) * 2 * D * D + (size_t)r * D + c0;
      __nv_bfloat16* lo = hi + D * D;
#pragma unroll
      for (int e = 0; e < 32; e += 8) {
        uint32_t h4[4], l4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const __nv_bfloat162 h = __floats2bfloat162_rn(m[e + 2 * q], m[e + 2 * q + 1]);
          const float2 hf = __bfloat1622float2(h);
          const __nv_bfloat162 l =
              __floats2bfloat162_rn(m[e + 2 * q] - hf.x, m[e + 2 * q + 1] - hf.y);
          h4[q] = *reinterpret_cast<const uint32_t*>(&h);
          l4[q] = *reinterpret_cast<const uint32_t*>(&l);
        }
        *reinterpret_cast<uint4*>(hi + e) = make_uint4(h4[0], h4[1], h4[2], h4[3]);
        *reinterpret_cast<uint4*>(lo + e) = make_uint4(l4[0], l4[1], l4[2], l4[3]);
      }
    };
    if (!delta) {
      // Linear: M_s = M_{s-1} + dM_s, with two segments' dM in flight (a and b hold
      // the even and odd segments)
      float a[32], b[32];
      if (S > 0) load_dm(a, 0);
      if (S > 1) load_dm(b, 1);
      for (int s = 0; s < S; s += 2) {
        emit(s);
#pragma unroll
        for (int e = 0; e < 32; ++e) m[e] += a[e];
        if (s + 2 < S) load_dm(a, s + 2);
        if (s + 1 < S) {
          emit(s + 1);
#pragma unroll
          for (int e = 0; e < 32; ++e) m[e] += b[e];
          if (s + 3 < S) load_dm(b, s + 3);
        }
      }
    } else {
      float nx[32];
      if (S > 0) load_dm(nx, 0);
      for (int s = 0; s < S; ++s) {
        emit(s);
        float dm[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) dm[e] = nx[e];
        if (s + 1 < S) load_dm(nx, s + 1);
        // M^T block (tf32) -> shared memory: row c, K-major, 4 boxes of 32 k
        const uint32_t kb = (uint32_t)(r >> 5), kin = (uint32_t)(r & 31);
#pragma unroll
        for (int cc = 0; cc < 32; ++cc) {
          const uint32_t off = kb * (32 * 128) + sw128((uint32_t)cc, kin >> 2) + (kin & 3) * 4;
          *reinterpret_cast<uint32_t*>(sMt + off) = tf32_rna(m[cc]);
        }
        fence_proxy_async_smem();
        mbar_arrive_warp(bar_mt);
        if (!mbar_wait_warp(bar_seg, (uint32_t)(s & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t gm[32];
        tmem_ld32(tmem_d + ((uint32_t)(warp * 32) << 16), gm);
        tmem_wait_ld();
        tc_fence_before();
#pragma unroll
        for (int e = 0; e < 32; ++e) m[e] += dm[e] - __uint_as_float(gm[e]);
      }
    }
    if (M_out && ok) {
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(M_out + ((size_t)bh * D + r) * D + c0 + e) =
            make_float4(m[e], m[e + 1], m[e + 2], m[e + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_d, 32);
  }
}

// prep_first_kernel: grid = (BH, 16), block 128; block y covers rows 8y .. 8y+7.
// Writes what the attention kernel reads for the first segment, M_{-1} = M_in as
// hi / lo bf16 and z_{-1} = z_in (zero when absent), exactly as chain_kernel and
// zscan_kernel would, so that a one-segment call can run the attention beside the
// state update; block (0, 0) also zeroes the counters of the kernels that follow.
__global__ void __launch_bounds__(D) prep_first_kernel(const float* M_in, const float* z_in,
                                                       __nv_bfloat16* __restrict__ Mhl,
                                                       float* __restrict__ zprev, int S,
                                                       unsigned* ctr, int nctr) {
  if (blockIdx.x == 0 && blockIdx.y == 0)
    for (int i = threadIdx.x; i < nctr; i += blockDim.x) ctr[i] = 0u;
  const int bh = blockIdx.x, r = blockIdx.y * 8 + (threadIdx.x >> 4), c = (threadIdx.x & 15) * 8;
  float m[8];
  if (M_in) {
    const float4* src = reinterpret_cast<const float4*>(M_in + ((size_t)bh * D + r) * D + c);
    const float4 a0 = src[0], a1 = src[1];
    m[0] = a0.x; m[1] = a0.y; m[2] = a0.z; m[3] = a0.w;
    m[4] = a1.x; m[5] = a1.y; m[6] = a1.z; m[7] = a1.w;
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) m[q] = 0.f;
  }
  uint32_t h4[4], l4[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(m[2 * q], m[2 * q + 1]);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(m[2 * q] - hf.x, m[2 * q + 1] - hf.y);
    h4[q] = *reinterpret_cast<const uint32_t*>(&h);
    l4[q] = *reinterpret_cast<const uint32_t*>(&l);
  }
  __nv_bfloat16* hi = Mhl + (size_t)bh * S * 2 * D * D + (size_t)r * D + c;
  *reinterpret_cast<uint4*>(hi) = make_uint4(h4[0], h4[1], h4[2], h4[3]);
  *reinterpret_cast<uint4*>(hi + D * D) = make_uint4(l4[0], l4[1], l4[2], l4[3]);
  if (blockIdx.y == 0) {
    const int f = threadIdx.x;
    zprev[(size_t)bh * S * D + f] = z_in ? z_in[(size_t)bh * D + f] : 0.f;
  }
}

}  // namespace

cudaError_t bf16_prep_first(const float* M_in, const float* z_in, const Bf16Workspace& ws,
                            int BH, int S, cudaStream_t stream, unsigned* ctr, int nctr) {
  prep_first_kernel<<<dim3(BH, D / 8), D, 0, stream>>>(M_in, z_in, ws.Mhl, ws.zprev, S, ctr,
                                                       nctr);
  return cudaGetLastError();
}

void bf16_state_plan(int BH, int S, int N, int* CH, int* CL) {
  // Chunk the segments so that the state GEMM has at least ~2 CTAs per SM, with
  // chunks of at least 128 tokens.
  const long long units = (long long)BH * S;
  int ch = 1;
  // At most 8 chunks: the chain adds each chunk's G M in turn (one segment's
  // chunks in sequence), which outweighs a more parallel state GEMM beyond that
  // (one-segment steps of 2048 tokens: 8 chunks 69 us per step, 16 chunks 75 us).
  const int maxch = N >= 128 ? (N / 128 < 8 ? N / 128 : 8) : 1;
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
                              int CL, int mode, int first, cudaStream_t stream,
                              const Bf16Layout* lay) {
  const unsigned nunits = (unsigned)((long long)BH * S * CH);
  // persistent: one CTA per SM walks the units (head, segment, token chunk)
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const unsigned grid = nunits < (unsigned)sms ? nunits : (unsigned)sms;
  // key/value head i = (batch row i / Hkv, head i % Hkv); without a layout, BH
  // contiguous [L, 128] planes
  const Bf16Layout l = lay ? *lay : Bf16Layout::bhld(BH, 1, L);
  const int Hkv = l.H_kv;
  CUtensorMap mk, mv;
  if (!make_bf16_map4(&mk, k, (uint64_t)L, Hkv, l.B, l.kv_sl, l.kv_sh, l.kv_sb, kSlab) ||
      !make_bf16_map4(&mv, v, (uint64_t)L, Hkv, l.B, l.kv_sl, l.kv_sh, l.kv_sb, kSlab))
    return cudaErrorInvalidValue;
  if (mode == 1 && !(first == 1 && S == 1)) {
    // Linear+Delta needs z_{s-1} (hence every segment's sum of sigma(K)) first
    zpart_kernel<<<nunits, 256, 0, stream>>>(k, ws.zpart, L, N, S, CH, CL, Hkv, l.kv_sb, l.kv_sh,
                                             l.kv_sl);
    zscan_kernel<<<BH, D, 0, stream>>>(ws.zpart, z_in, z_out, ws.zprev, S, CH, first);
    state_kernel<<<grid, kStateThreads, kStateSmem, stream>>>(
        mk, mv, ws.zprev, ws.dpart, ws.zpart, L, N, S, CH, CL, mode, 0, Hkv, (long long)nunits);
  } else {
    // The state GEMM also produces the sums of sigma(K): always in Linear mode, and
    // in Linear+Delta mode for a lone segment whose z_{-1} is already in place. In
    // Linear mode the chain kernel scans z itself.
    state_kernel<<<grid, kStateThreads, kStateSmem, stream>>>(
        mk, mv, ws.zprev, ws.dpart, ws.zpart, L, N, S, CH, CL, mode, 1, Hkv, (long long)nunits);
    if (mode == 1)
      zscan_kernel<<<BH, D, 0, stream>>>(ws.zpart, z_in, z_out, ws.zprev, S, CH, first);
  }
  CUtensorMap mg;
  if (mode == 1) {
    // G planes of dpart, fp32 [planes][128][128]; box 32 columns x 128 rows
    EncodeTiledFn enc = get_encode_fn();
    const cuuint64_t dims[3] = {128, 128, (cuuint64_t)nunits * 2};
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
  const bool fused_z = mode == 0;
  chain_kernel<<<dim3(BH, 4), kChainThreads, kChainSmem, stream>>>(
      mg, ws.dpart, M_in, M_out, ws.Mhl, S, CH, mode, first, fused_z ? ws.zpart : nullptr,
      z_in, z_out, ws.zprev);
  return cudaGetLastError();
}

}  // namespace infini
