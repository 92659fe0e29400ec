// bf16_step_state.cu — the memory update of a call that holds one segment (every
// streaming step), bf16 k/v, d = 128.
//
// With one segment the incoming state (M_in, z_in) is known before the call, so the
// Linear+Delta rule of "Leave No Context Behind" (arXiv 2404.07143, as quoted on
// llm-papers-study.pages.dev, section 3.4) is evaluated in the pages' own order:
//   R   = sigma(K) M_in / (sigma(K) z_in)     row by row (0 where the denominator is 0)
//   M   = M_in + sigma(K)^T (V - R),   z = z_in + sum_t sigma(K_t)
// (Linear: R = 0). Every term of the sum over tokens is independent, so the tokens are
// cut into chunks processed in parallel, and the value columns into two blocks of 64
// (column block j of M needs only column block j of M_in, V and R). One CTA per
// (head, token chunk, column block) computes its chunk's sigma(K)^T (V - R) for its
// columns on the tensor cores; the last CTA of each (head, column block) to finish
// adds the chunks' partial sums to M_in in chunk order (the result does not depend on
// which CTA finishes last) and writes M_out; the column block 0 CTAs also sum z.
// No sequential chain and no d x d x d product remain.
//
// Precision: sigma(K) = hi + lo, M_in = hi + lo and V - R = hi + lo as bf16 pairs;
// each product keeps the three terms above 2^-16 relative (hi hi, hi lo, lo hi), with
// fp32 accumulation: ~2^-16 relative per term, as the multi-segment state GEMM.
//
// Roles (576 threads): warps 0-15 convert (sigma(K) hi/lo and 1/den per token, then
// U = V - R/den as hi/lo) in two groups of eight, group g taking the slabs of stage g,
// so that two slabs are converted at once; warp 16 issues the TMA copies, warp 17
// allocates tensor memory and issues the MMAs. Tokens move in slabs of 128 through two
// stages:
//   K [128 tokens x 128 features] bf16 (two 64-feature boxes), overwritten by sigma(K)_hi
//   KL  sigma(K)_lo, same layout
//   V [128 tokens x 64 columns] bf16, overwritten by U_hi;  UL  U_lo
// Tensor memory: R of each stage [128 tokens x 64] (columns 0-63, 64-127) and the
// chunk's sum [128 features x 64] (columns 128-191).
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "bf16_path.h"
#include "sm100.cuh"
#include "tma_map.h"

namespace infini {
namespace {

constexpr int D = 128;
constexpr int kCols = 64;                    // value columns per CTA
constexpr int kCB = D / kCols;               // column blocks
constexpr int kSlab = 128;                   // tokens per slab
constexpr int kBox = kSlab * 128;            // one [128 x 64] bf16 box: 16 KB
constexpr int OFF_MH = 0, OFF_ML = kBox;     // M_in[:, block] hi / lo [128 features x 64]
constexpr int OFF_STAGE = 2 * kBox;
constexpr int S_K = 0, S_KL = 2 * kBox, S_V = 4 * kBox, S_UL = 5 * kBox;
constexpr int kStageBytes = 6 * kBox;        // 96 KB
constexpr int kStages = 2;
constexpr int OFF_INV = OFF_STAGE + kStages * kStageBytes;  // [2][128] f32
constexpr int OFF_BAR = OFF_INV + kStages * kSlab * 4;
constexpr int kSmem = OFF_BAR + 256 + 1024;  // + alignment slack
constexpr int kGroupWarps = 8;                // converter warps per group (one group per stage)
constexpr int kConvWarps = 2 * kGroupWarps;
constexpr int kConvThreads = kConvWarps * 32;
constexpr int kThreads = (kConvWarps + 2) * 32;
constexpr int kProdWarp = kConvWarps, kMmaWarp = kConvWarps + 1;

enum {
  B_FULL = 0 /* 2 */, B_CONV1 = 2 /* 2 */, B_RDONE = 4 /* 2 */, B_CONV2 = 6 /* 2 */,
  B_FREE = 8 /* 2 */, B_MFULL = 10, B_DONE = 11, B_COUNT = 12
};

// K-major operand (rows = M index, 128 bytes = 64 bf16 of K per row in each of two boxes
// kBox apart): k-step kk covers K elements [16 kk, 16 kk + 16).
__device__ __forceinline__ uint64_t kmajor(uint32_t base, int kk) {
  return sdesc(base + (uint32_t)(kk >> 2) * kBox + (uint32_t)(kk & 3) * 32, 16, 1024);
}
// MN-major operand (rows = K index, 128 bytes of M or N per row, 64-element chunks kBox
// apart): k-step kk covers K rows [16 kk, 16 kk + 16).
__device__ __forceinline__ uint64_t mnmajor(uint32_t base, int kk) {
  return sdesc(base + (uint32_t)kk * 2048, kBox, 1024);
}

__device__ __forceinline__ void split_bf16(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Bounded wait used only while draining after an error: ignores the error flag.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) break;  // 200 ms
  }
}

struct StepParams {
  int N;          // tokens of the segment
  int CH, CL;     // token chunks per head and tokens per chunk (a multiple of kSlab)
  int Hkv;        // key/value heads per batch row (head index bh = b * Hkv + h)
  int delta;
  const float* zprev;   // [BH][128]: z_in (the copy the call made before forking)
  const float* M_in;    // [BH][128][128] or NULL (zero state)
  float* M_out;         // [BH][128][128]
  float* z_out;         // [BH][128]
  float* part;          // [BH][kCB][CH] records of 128 x 64 partial sums (2048 float4)
  float* zpart;         // [BH][CH][128]
  unsigned* ctr;        // [BH][kCB] chunks finished (zeroed before the launch)
};

__global__ void __launch_bounds__(kThreads, 1)
step_state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_m, const StepParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  float* sInv = reinterpret_cast<float*>(smem + OFF_INV);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + B_COUNT);
  int* sLast = reinterpret_cast<int*>(tmem_slot + 1);

  const int cb = blockIdx.x % kCB;
  const int c = (blockIdx.x / kCB) % p.CH;
  const int bh = blockIdx.x / (kCB * p.CH);
  const int beg = min(p.N, c * p.CL), end = min(p.N, (c + 1) * p.CL);
  const int len = end - beg;
  const int nslab = (len + kSlab - 1) / kSlab;
  const bool delta = p.delta != 0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars[B_FULL + s], 1);
      mbar_init(&bars[B_CONV1 + s], kGroupWarps);
      mbar_init(&bars[B_RDONE + s], 1);
      mbar_init(&bars[B_CONV2 + s], kGroupWarps);
      mbar_init(&bars[B_FREE + s], 1);
    }
    mbar_init(&bars[B_MFULL], 1);
    mbar_init(&bars[B_DONE], 1);
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tDM = tmem + 128;
  bool ok = true;

  if (warp == kProdWarp) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      const int hk = bh % p.Hkv, b = bh / p.Hkv;
      int issued[kStages] = {0, 0};
      if (delta) {
        mbar_arrive_expect_tx(&bars[B_MFULL], 2 * kBox);
        tma_load_3d(smem + OFF_MH, &tm_m, &bars[B_MFULL], cb * kCols, 0, bh * 2);
        tma_load_3d(smem + OFF_ML, &tm_m, &bars[B_MFULL], cb * kCols, 0, bh * 2 + 1);
      }
      for (int n = 0; n < nslab && ok; ++n) {
        const int st = n & 1;
        if (n >= kStages && !mbar_wait(&bars[B_FREE + st], (uint32_t)(((n >> 1) - 1) & 1))) {
          ok = false;
          break;
        }
        uint8_t* sb = smem + OFF_STAGE + st * kStageBytes;
        const int row = beg + n * kSlab;
        mbar_arrive_expect_tx(&bars[B_FULL + st], 3 * kBox);
        tma_load_4d(sb + S_K, &tm_k, &bars[B_FULL + st], 0, row, hk, b);
        tma_load_4d(sb + S_K + kBox, &tm_k, &bars[B_FULL + st], 64, row, hk, b);
        tma_load_4d(sb + S_V, &tm_v, &bars[B_FULL + st], cb * kCols, row, hk, b);
        ++issued[st];
      }
      if (!ok) {  // let the copies already issued land before the CTA exits
        if (delta) drain_wait(&bars[B_MFULL], 0);
        for (int st = 0; st < kStages; ++st)
          if (issued[st] > 0) drain_wait(&bars[B_FULL + st], (uint32_t)((issued[st] - 1) & 1));
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer (whole warp waits, one elected lane issues) ----------------
    // Linear+Delta order: R(n) as soon as slab n is converted, then the update product of
    // slab n - 1 (whose U the other converter group has formed meanwhile).
    const uint32_t id_r = idesc_f32acc(1, 0, 1, 128, kCols);   // sigma(K) [K-major] x M [MN-major]
    const uint32_t id_m = idesc_f32acc(1, 1, 1, 128, kCols);   // sigma(K)^T [MN] x U [MN]
    if (delta && nslab > 0) ok = mbar_wait_warp(&bars[B_MFULL], 0);
    tc_fence_after();
    const uint32_t mh = smem_u32(smem + OFF_MH), ml = smem_u32(smem + OFF_ML);
    auto update = [&](int n) {  // sum += sigma(K)^T U over slab n's tokens
      const int st = n & 1;
      const uint32_t sb = smem_u32(smem + OFF_STAGE + st * kStageBytes);
      const uint32_t kh = sb + S_K, kl = sb + S_KL, uh = sb + S_V, ul = sb + S_UL;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kSlab / 16; ++kk) {
          const uint32_t acc = (n > 0 || kk > 0) ? 1u : 0u;
          mma_bf16_ss(tDM, mnmajor(kh, kk), mnmajor(uh, kk), id_m, acc);
          if (delta) mma_bf16_ss(tDM, mnmajor(kh, kk), mnmajor(ul, kk), id_m, 1u);
          mma_bf16_ss(tDM, mnmajor(kl, kk), mnmajor(uh, kk), id_m, 1u);
        }
        mma_commit(&bars[B_FREE + st]);
      }
      __syncwarp();
    };
    auto wait_u = [&](int n) {  // U of slab n formed (Linear+Delta)
      return mbar_wait_warp(&bars[B_CONV2 + (n & 1)], (uint32_t)((n >> 1) & 1));
    };
    for (int n = 0; n < nslab && ok; ++n) {
      const int st = n & 1;
      if (!mbar_wait_warp(&bars[B_CONV1 + st], (uint32_t)((n >> 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (!delta) {  // U = V, exact in bf16
        update(n);
        continue;
      }
      // R = sigma(K) M_in for the slab's tokens (rows) and this CTA's 64 columns
      const uint32_t sb = smem_u32(smem + OFF_STAGE + st * kStageBytes);
      const uint32_t kh = sb + S_K, kl = sb + S_KL;
      const uint32_t tR = tmem + (uint32_t)st * kCols;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          mma_bf16_ss(tR, kmajor(kh, kk), mnmajor(mh, kk), id_r, kk > 0 ? 1u : 0u);
          mma_bf16_ss(tR, kmajor(kh, kk), mnmajor(ml, kk), id_r, 1u);
          mma_bf16_ss(tR, kmajor(kl, kk), mnmajor(mh, kk), id_r, 1u);
        }
        mma_commit(&bars[B_RDONE + st]);
      }
      __syncwarp();
      if (n > 0) {
        if (!wait_u(n - 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        update(n - 1);
      }
    }
    if (ok && delta && nslab > 0) {
      ok = wait_u(nslab - 1);
      tc_fence_after();
      if (ok) update(nslab - 1);
    }
    if (elect_one()) mma_commit(&bars[B_DONE]);  // tracks every MMA issued above
    __syncwarp();
  } else {
    // ---------------- converters: two groups of 8 warps, group g takes the slabs of stage g
    const int grp = warp / kGroupWarps, lw = warp % kGroupWarps;
    // Phase 1, a warp per token row at a time: lane l holds features [4l, 4l + 4).
    float zr[4], zs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int e = 0; e < 4; ++e) zr[e] = delta ? p.zprev[(size_t)bh * D + 4 * lane + e] : 0.f;
    const uint32_t fbox = (uint32_t)(lane >> 4) * kBox;      // features 0-63 / 64-127
    const uint32_t funit = (uint32_t)((lane & 15) >> 1);      // 16-byte unit in the row
    const uint32_t fhalf = (uint32_t)(lane & 1) * 8;          // 8-byte half of the unit
    for (int n = grp; n < nslab && ok; n += kStages) {
      const int st = n & 1;
      const uint32_t par = (uint32_t)((n >> 1) & 1);
      uint8_t* sb = smem + OFF_STAGE + st * kStageBytes;
      float* inv = sInv + st * kSlab;
      if (!mbar_wait_warp(&bars[B_FULL + st], par)) {
        ok = false;
        break;
      }
      // rows t = lw + 8 j: eight rows at a time, so that their loads, exponentials and
      // stores overlap instead of forming one dependent chain per row
#pragma unroll
      for (int g = 0; g < kSlab / (kGroupWarps * 8); ++g) {
        float dp[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int t = lw + kGroupWarps * (8 * g + j);
          const bool valid = n * kSlab + t < len;
          const uint32_t off =
              fbox + (uint32_t)t * 128u + ((funit ^ (uint32_t)(t & 7)) << 4) + fhalf;
          const uint2 raw = *reinterpret_cast<const uint2*>(sb + S_K + off);
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
          const float2 x01 = __bfloat1622float2(h2[0]), x23 = __bfloat1622float2(h2[1]);
          float f[4] = {elu1(x01.x), elu1(x01.y), elu1(x23.x), elu1(x23.y)};
          float den = 0.f;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            f[e] = valid ? f[e] : 0.f;  // rows past the segment: sigma(K) = 0, no term
            zs[e] += f[e];
            den = fmaf(f[e], zr[e], den);
          }
          dp[j] = den;
          uint2 hi, lo;
          split_bf16(f[0], f[1], hi.x, lo.x);
          split_bf16(f[2], f[3], hi.y, lo.y);
          *reinterpret_cast<uint2*>(sb + S_K + off) = hi;
          *reinterpret_cast<uint2*>(sb + S_KL + off) = lo;
        }
        if (delta) {
          // sum each row's 32 lane partials: a transposed reduction (lane bits 4, 3, 2
          // pick the rows a lane keeps, bits 1, 0 finish the sum), after which lane l
          // holds row j = (l >> 2) & 7 of the eight
          const bool b4 = (lane >> 4) & 1, b3 = (lane >> 3) & 1, b2 = (lane >> 2) & 1;
          float v4[4], v2[2];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float keep = b4 ? dp[k + 4] : dp[k], give = b4 ? dp[k] : dp[k + 4];
            v4[k] = keep + __shfl_xor_sync(0xffffffffu, give, 16);
          }
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const float keep = b3 ? v4[k + 2] : v4[k], give = b3 ? v4[k] : v4[k + 2];
            v2[k] = keep + __shfl_xor_sync(0xffffffffu, give, 8);
          }
          float v1 = (b2 ? v2[1] : v2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? v2[0] : v2[1], 4);
          v1 += __shfl_xor_sync(0xffffffffu, v1, 2);
          v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
          if ((lane & 3) == 0) {
            const int t = lw + kGroupWarps * (8 * g + ((lane >> 2) & 7));
            inv[t] = v1 != 0.f ? 1.f / v1 : 0.f;
          }
        }
      }
      fence_proxy_async_smem();
      mbar_arrive_warp(&bars[B_CONV1 + st]);
      if (!delta) continue;
      // Phase 2 (Linear+Delta): U = V - R / den for token r (tensor-memory lane) and 32
      // of the block's columns; V is overwritten by U_hi, U_lo goes beside it. The
      // first wait orders every warp's 1/den writes of the group before these reads.
      if (!mbar_wait_warp(&bars[B_CONV1 + st], par) ||
          !mbar_wait_warp(&bars[B_RDONE + st], par)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int r = (warp & 3) * 32 + lane;
      const int ch = lw >> 2;  // columns [32 ch, 32 ch + 32)
      uint32_t rr[32];
      tmem_ld32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(st * kCols + 32 * ch), rr);
      tmem_wait_ld();
      const float iv = inv[r];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t off = sw128((uint32_t)r, (uint32_t)(4 * ch + u));
        const uint4 vraw = *reinterpret_cast<const uint4*>(sb + S_V + off);
        const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&vraw);
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 vv = __bfloat1622float2(v2[e]);
          const float u0 = vv.x - __uint_as_float(rr[8 * u + 2 * e]) * iv;
          const float u1 = vv.y - __uint_as_float(rr[8 * u + 2 * e + 1]) * iv;
          split_bf16(u0, u1, hi[e], lo[e]);
        }
        *reinterpret_cast<uint4*>(sb + S_V + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(sb + S_UL + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive_warp(&bars[B_CONV2 + st]);
    }
    // Every product issued must be done before tensor memory is read or freed, also
    // after an error (the MMA warp commits B_DONE in every case).
    if (ok) ok = mbar_wait_warp(&bars[B_DONE], 0);
    if (!ok) drain_wait(&bars[B_DONE], 0);
    tc_fence_after();
    // the chunk's sum of sigma(K): lane l of every converter warp holds features [4l, 4l + 4)
    float* red = reinterpret_cast<float*>(smem + OFF_STAGE);  // the stages are idle now
#pragma unroll
    for (int e = 0; e < 4; ++e) red[warp * D + 4 * lane + e] = zs[e];
    if (warp < kGroupWarps) {
      // the chunk's partial sum of sigma(K)^T U for this block's columns -> its record,
      // laid out [half ch][column quad q][feature f] float4 so that a warp writes 512
      // contiguous bytes per instruction, and the summing CTA reads them the same way
      const int f = (warp & 3) * 32 + lane;  // feature (tensor-memory lane)
      const int ch = warp >> 2;
      uint32_t dm[32];
      if (nslab > 0) {
        tmem_ld32(tDM + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(32 * ch), dm);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) dm[e] = 0u;
      }
      float4* rec = reinterpret_cast<float4*>(p.part) + (((size_t)bh * kCB + cb) * p.CH + c) * 2048;
#pragma unroll
      for (int q = 0; q < 8; ++q)
        __stcg(rec + (ch * 8 + q) * 128 + f,
               make_float4(__uint_as_float(dm[4 * q]), __uint_as_float(dm[4 * q + 1]),
                           __uint_as_float(dm[4 * q + 2]), __uint_as_float(dm[4 * q + 3])));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (cb == 0 && tid < D) {
    const float* red = reinterpret_cast<const float*>(smem + OFF_STAGE);
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kConvWarps; ++w) s += red[w * D + tid];
    __stcg(p.zpart + ((size_t)bh * p.CH + c) * D + tid, s);
  }
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
  // The last CTA of (head, column block) to finish adds the chunks' sums in chunk order.
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned done = atomicAdd(p.ctr + bh * kCB + cb, 1u);
    *sLast = (done == (unsigned)p.CH - 1u) && !device_error_set() ? 1 : 0;
  }
  __syncthreads();
  if (!*sLast) return;
  __threadfence();
  if (tid < kConvThreads) {
    // thread tid takes the record's float4 number u * 512 + tid for u = 0..3: feature row
    // f = index & 127, columns 32 (index >> 10) + 4 ((index >> 7) & 7) of the block
    float4 acc[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = u * kConvThreads + tid, f = idx & 127;
      const int col = cb * kCols + 32 * (idx >> 10) + 4 * ((idx >> 7) & 7);
      acc[u] = p.M_in ? *reinterpret_cast<const float4*>(p.M_in + ((size_t)bh * D + f) * D + col)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const float4* rec0 = reinterpret_cast<const float4*>(p.part) + (((size_t)bh * kCB + cb) * p.CH) * 2048;
    // two chunks per round so that eight loads are in flight; the chunks are still
    // added to acc in chunk order
    for (int cc = 0; cc < p.CH; cc += 2) {
      float4 a[2][4];
#pragma unroll
      for (int k = 0; k < 2; ++k)
#pragma unroll
        for (int u = 0; u < 4; ++u)
          a[k][u] = cc + k < p.CH ? __ldcg(rec0 + (size_t)(cc + k) * 2048 + u * kConvThreads + tid)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < 2; ++k)
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          acc[u].x += a[k][u].x;
          acc[u].y += a[k][u].y;
          acc[u].z += a[k][u].z;
          acc[u].w += a[k][u].w;
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = u * kConvThreads + tid, f = idx & 127;
      const int col = cb * kCols + 32 * (idx >> 10) + 4 * ((idx >> 7) & 7);
      *reinterpret_cast<float4*>(p.M_out + ((size_t)bh * D + f) * D + col) = acc[u];
    }
    if (cb == 0 && tid < D) {
      float z = p.zprev[(size_t)bh * D + tid];
      const float* zp = p.zpart + (size_t)bh * p.CH * D + tid;
      for (int cc = 0; cc < p.CH; cc += 4) {
        float t4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) t4[e] = cc + e < p.CH ? __ldcg(zp + (size_t)(cc + e) * D) : 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) z += t4[e];
      }
      p.z_out[(size_t)bh * D + tid] = z;
    }
  }
}

}  // namespace

cudaError_t bf16_step_state_set_attributes() {
  return cudaFuncSetAttribute(step_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kSmem);
}

void bf16_step_state_plan(int BH, int N, int* CH, int* CL) {
  // about 64 CTAs (the attention kernel of the same call takes the other SMs, and all
  // of them as these free up), chunks of whole slabs, at most 16 chunks per head
  const int nslab = (N + kSlab - 1) / kSlab;
  int ch = (64 + BH * kCB - 1) / (BH * kCB);
  ch = max(1, min(min(ch, 16), nslab));
  const int per = (nslab + ch - 1) / ch;
  *CL = per * kSlab;
  *CH = (nslab + per - 1) / per;
}

size_t bf16_step_state_bytes(int BH, int CH) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return up((size_t)BH * kCB * CH * D * kCols * 4) + up((size_t)BH * CH * D * 4) +
         up((size_t)BH * kCB * 4);
}

cudaError_t bf16_step_state_launch(const __nv_bfloat16* k, const __nv_bfloat16* v,
                                   const float* M_in, float* M_out, float* z_out,
                                   const Bf16Workspace& ws, void* step_ws, int BH, int N, int CH,
                                   int CL, int mode, cudaStream_t stream, const Bf16Layout* lay) {
  const Bf16Layout l = lay ? *lay : Bf16Layout::bhld(BH, 1, N);
  CUtensorMap mk, mv, mm;
  if (!make_bf16_map4(&mk, k, (uint64_t)N, l.H_kv, l.B, l.kv_sl, l.kv_sh, l.kv_sb, kSlab) ||
      !make_bf16_map4(&mv, v, (uint64_t)N, l.H_kv, l.B, l.kv_sl, l.kv_sh, l.kv_sb, kSlab) ||
      !make_bf16_map(&mm, ws.Mhl, D, (uint64_t)BH * 2, 128))
    return cudaErrorInvalidValue;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  StepParams p;
  p.N = N;
  p.CH = CH;
  p.CL = CL;
  p.Hkv = l.H_kv;
  p.delta = mode == 1 ? 1 : 0;
  p.zprev = ws.zprev;
  p.M_in = M_in;
  p.M_out = M_out;
  p.z_out = z_out;
  char* base = static_cast<char*>(step_ws);
  p.part = reinterpret_cast<float*>(base);
  base += up((size_t)BH * kCB * CH * D * kCols * 4);
  p.zpart = reinterpret_cast<float*>(base);
  base += up((size_t)BH * CH * D * 4);
  p.ctr = reinterpret_cast<unsigned*>(base);
  step_state_kernel<<<(unsigned)(BH * CH * kCB), kThreads, kSmem, stream>>>(mk, mv, mm, p);
  return cudaGetLastError();
}

unsigned* bf16_step_state_counters(void* step_ws, int BH, int CH) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return reinterpret_cast<unsigned*>(static_cast<char*>(step_ws) +
                                     up((size_t)BH * kCB * CH * D * kCols * 4) +
                                     up((size_t)BH * CH * D * 4));
}

}  // namespace infini
