// bf16_decode.cu — token-level streaming decode (bf16, d = 128).
//
// n new tokens of every (batch, head) join the current segment, whose first `pos`
// tokens sit in the caller's KV cache. Token t = pos + i of the segment attends
// causally to cache rows 0..t and retrieves from the memory of the segments before
// it ("Leave No Context Behind", arXiv 2404.07143, as quoted on
// llm-papers-study.pages.dev: sections 3.1 (dot-product attention), 3.3 (retrieval
// sigma(Q) M_{s-1} / sigma(Q) z_{s-1}), 3.5 (gate); the per-segment streaming is the
// same section's "fast streaming inference"). The result for every token is the
// one the whole-sequence forward gives it.
//
// The work is a batch of short matrix-vector products over the cache: it is bound
// by reading the cache (512 B per cached token-head) and the fp32 memory (64 KiB per
// head), so it runs on CUDA cores, split over the cache like flash decoding:
//   decode_partial_kernel  grid (splits, BH, query groups of up to 16). A CTA stages
//                          64-row chunks of K and V in shared memory (16-byte loads,
//                          coalesced): cache rows below pos from the cache, the new
//                          rows straight from the call's k and v (the last query
//                          group also writes those into the cache; nothing in the
//                          call reads them from there). It scores every query of
//                          its group against the chunk (two threads per row, 64
//                          features each) and keeps one online-softmax partial
//                          (max, sum, 128 accumulators) per query in exp2 units.
//                          One more CTA per (head, group) computes the retrieval
//                          sigma(q) M_{s-1} (a column per thread, M read
//                          row-coalesced) and sigma(q) z_{s-1}, beside the cache reads.
//   decode_combine_kernel  grid (BH, queries). Merges the splits' partials of one
//                          query, divides the retrieval by its denominator, applies
//                          the gate and writes out in bf16.
// The partial kernel is compiled for query-group widths 1, 2, 4, 8 and 16, so a
// single token carries no idle accumulators.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "bf16_path.h"
#include "sm100.cuh"

namespace infini {
namespace {

constexpr int D = 128;
constexpr int kRows = 64;     // cache rows per chunk
constexpr int kGroup = 16;    // queries per CTA
constexpr int kThreads = 128;
constexpr int kPart = 2 + D;  // one partial: max, sum, 128 accumulators
constexpr int kMaxSplits = 512;
constexpr int kRetCTAs = 1;   // retrieval CTAs per (head, group): thread t forms column t
constexpr int kRet = D + 1;   // one retrieval record: sigma(q) M (128), sigma(q) z

struct DecodeParams {
  int n, pos, N, H, splits, chunks_per_split, groups;
};

__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

template <int NQ>
__global__ void __launch_bounds__(kThreads, 4)  // four CTAs per SM (shared memory allows four)
decode_partial_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ knew,
                      const __nv_bfloat16* __restrict__ vnew, __nv_bfloat16* __restrict__ kc,
                      __nv_bfloat16* __restrict__ vc, const float* __restrict__ M,
                      const float* __restrict__ z, float* __restrict__ part,
                      float* __restrict__ ret, const DecodeParams p) {
  __shared__ __align__(16) float sq[kGroup][D];    // queries, scaled by log2(e) / sqrt(d)
  __shared__ __align__(16) uint32_t sk[kRows][D / 2];  // bf16 pairs
  __shared__ __align__(16) uint32_t sv[kRows][D / 2];
  __shared__ float ss[kGroup][kRows];              // scores, then probabilities
  __shared__ float sm_m[kGroup], sm_l[kGroup], sm_a[kGroup];

  const int split = blockIdx.x, bh = blockIdx.y, grp = blockIdx.z;
  const int t = threadIdx.x;
  const int q0 = grp * kGroup;
  const int nq = min(kGroup, p.n - q0);
  const float sl = 1.4426950408889634f * 0.08838834764831845f;  // log2(e) / sqrt(128)

  if (split >= p.splits) {
    // the retrieval CTA: thread t forms column t of sigma(q) M_{s-1} (M read
    // row-coalesced, 32 rows' loads in flight), and the CTA the denominators
    // sigma(q) z_{s-1}. One such CTA per (head, group) keeps a one-token call within
    // one wave of CTAs beside the cache splits.
    const int lane = t & 31, w = t >> 5;
    float (*sphi)[D] = sq;
    for (int i = 0; i < nq; ++i)
      sphi[i][t] = elu1(__bfloat162float(q[((size_t)bh * p.n + q0 + i) * D + t]));
    __syncthreads();
    float* rec = ret + ((size_t)bh * p.groups + grp) * kGroup * kRet;
    const float zt = z[(size_t)bh * D + t];
    for (int i = 0; i < nq; ++i) {
      float dp = sphi[i][t] * zt;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dp += __shfl_xor_sync(0xffffffffu, dp, o);
      if (lane == 0) ss[i][w] = dp;
    }
    float acc[NQ];
#pragma unroll
    for (int i = 0; i < NQ; ++i) acc[i] = 0.f;
    const float* Mc = M + (size_t)bh * D * D + t;
#pragma unroll 32
    for (int k = 0; k < D; ++k) {
      const float m = __ldg(Mc + (size_t)k * D);
#pragma unroll
      for (int i = 0; i < NQ; ++i)
        if (i < nq) acc[i] = fmaf(sphi[i][k], m, acc[i]);
    }
#pragma unroll
    for (int i = 0; i < NQ; ++i)
      if (i < nq) rec[i * kRet + t] = acc[i];
    __syncthreads();
    if (t < nq) rec[t * kRet + D] = (ss[t][0] + ss[t][1]) + (ss[t][2] + ss[t][3]);
    return;
  }

  for (int i = 0; i < nq; ++i)
    sq[i][t] = __bfloat162float(q[((size_t)bh * p.n + q0 + i) * D + t]) * sl;
  if (t < kGroup) {
    sm_m[t] = -INFINITY;
    sm_l[t] = 0.f;
  }
  // rows this group may see: query q0 + i sees rows 0 .. pos + q0 + i
  const int rows = p.pos + q0 + nq;
  const int r_begin = split * p.chunks_per_split * kRows;
  const int r_end = min(rows, r_begin + p.chunks_per_split * kRows);
  float acc[NQ];
#pragma unroll
  for (int i = 0; i < NQ; ++i) acc[i] = 0.f;
  const bool writer = grp == p.groups - 1;  // this group loads every new row

  const size_t base = (size_t)bh * p.N * D;
  for (int r0 = r_begin; r0 < r_end; r0 += kRows) {
    const int nr = min(kRows, r_end - r0);
    __syncthreads();  // the previous chunk's readers are done
    // K and V rows [r0, r0 + nr): 16 bytes per thread per step, row-contiguous
    // asynchronous 16-byte copies, all in flight before one wait
#pragma unroll
    for (int it = 0; it < kRows * (D / 8) / kThreads; ++it) {
      const int e = t + it * kThreads;
      const int row = e / (D / 8), c = e % (D / 8);
      const int R = r0 + row;
      if (row < nr) {
        const __nv_bfloat16* ks;
        const __nv_bfloat16* vs;
        if (R < p.pos) {
          ks = kc + base + (size_t)R * D + c * 8;
          vs = vc + base + (size_t)R * D + c * 8;
        } else {
          const size_t src = ((size_t)bh * p.n + (R - p.pos)) * D + c * 8;
          ks = knew + src;
          vs = vnew + src;
        }
        cp_async16(&sk[row][(c ^ (row & 15)) * 4], ks);
        cp_async16(&sv[row][c * 4], vs);
      }
    }
    cp_async_wait_all();
    __syncthreads();
    // the last group also writes the new rows it staged into the caches
    if (writer && r0 + nr > p.pos) {
      const int first = max(0, p.pos - r0);
      for (int e = first * (D / 8) + t; e < nr * (D / 8); e += kThreads) {
        const int row = e / (D / 8), c = e % (D / 8);
        const size_t dst = base + (size_t)(r0 + row) * D + c * 8;
        *reinterpret_cast<uint4*>(kc + dst) =
            *reinterpret_cast<const uint4*>(&sk[row][(c ^ (row & 15)) * 4]);
        *reinterpret_cast<uint4*>(vc + dst) = *reinterpret_cast<const uint4*>(&sv[row][c * 4]);
      }
    }
    // scores: thread (row r, part p). With 16 queries part p takes queries [8p, 8p + 8)
    // over all 128 features; with fewer, every query over features [64p, 64p + 64),
    // and the two parts' sums meet in shared memory. A warp's lanes are 32 rows with
    // the same part, so every query read is a broadcast; the rows' 16-byte chunks are
    // stored permuted (chunk c of row r at c ^ (r & 15)), so that the 32 rows' chunk c
    // fall in distinct banks.
    {
      constexpr int QPT = NQ == kGroup ? kGroup / 2 : NQ;  // queries per thread
      const int r = t & (kRows - 1), pt = t >> 6;
      const int qb = NQ == kGroup ? QPT * pt : 0;
      const int cb = NQ == kGroup ? 0 : 8 * pt, ce = NQ == kGroup ? D / 8 : 8 * pt + 8;
      float sc[QPT];
#pragma unroll
      for (int i = 0; i < QPT; ++i) sc[i] = 0.f;
      if (r < nr) {
#pragma unroll 2
        for (int c = cb; c < ce; ++c) {
          const uint4 kr = *reinterpret_cast<const uint4*>(&sk[r][(c ^ (r & 15)) * 4]);
          const float k8[8] = {bf_lo(kr.x), bf_hi(kr.x), bf_lo(kr.y), bf_hi(kr.y),
                               bf_lo(kr.z), bf_hi(kr.z), bf_lo(kr.w), bf_hi(kr.w)};
#pragma unroll
          for (int i = 0; i < QPT; ++i) {
            if (qb + i < nq) {
              const float4 qa = *reinterpret_cast<const float4*>(&sq[qb + i][8 * c]);
              const float4 qc = *reinterpret_cast<const float4*>(&sq[qb + i][8 * c + 4]);
              float v = fmaf(qa.x, k8[0], sc[i]);
              v = fmaf(qa.y, k8[1], v);
              v = fmaf(qa.z, k8[2], v);
              v = fmaf(qa.w, k8[3], v);
              v = fmaf(qc.x, k8[4], v);
              v = fmaf(qc.y, k8[5], v);
              v = fmaf(qc.z, k8[6], v);
              sc[i] = fmaf(qc.w, k8[7], v);
            }
          }
        }
      }
      if (NQ != kGroup && pt == 1) {
#pragma unroll
        for (int i = 0; i < QPT; ++i)
          if (i < nq) ss[i][r] = sc[i];
      }
      __syncthreads();
      if (NQ == kGroup || pt == 0) {
#pragma unroll
        for (int i = 0; i < QPT; ++i) {
          const int qi = qb + i;
          if (qi < nq) {
            const float v = NQ == kGroup ? sc[i] : sc[i] + ss[qi][r];
            ss[qi][r] = (r < nr && r0 + r <= p.pos + q0 + qi) ? v : -INFINITY;
          }
        }
      }
    }
    __syncthreads();
    // online softmax: eight threads per query, eight rows each
    {
      const int i = t >> 3, part8 = t & 7;
      float mx = -INFINITY;
      if (i < nq)
        for (int r = part8; r < kRows; r += 8) mx = fmaxf(mx, r < nr ? ss[i][r] : -INFINITY);
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float m_old = -INFINITY, m_new = -INFINITY, sum = 0.f;
      if (i < nq) {
        m_old = sm_m[i];
        m_new = fmaxf(m_old, mx);
        for (int r = part8; r < kRows; r += 8) {
          const float pr = (r < nr && m_new != -INFINITY) ? exp2f(ss[i][r] - m_new) : 0.f;
          ss[i][r] = pr;
          sum += pr;
        }
      }
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      __syncwarp();
      if (i < nq && part8 == 0) {
        const float a = m_new == -INFINITY ? 1.f : exp2f(m_old - m_new);
        sm_a[i] = a;
        sm_m[i] = m_new;
        sm_l[i] = sm_l[i] * a + sum;
      }
    }
    __syncthreads();
    // P V: thread t owns feature t
    {
#pragma unroll
      for (int i = 0; i < NQ; ++i)
        if (i < nq) acc[i] *= sm_a[i];
      // four rows per step: each query's four probabilities are one 128-bit broadcast
      int r = 0;
      for (; r + 4 <= nr; r += 4) {
        float vf[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t u = sv[r + k][t >> 1];
          vf[k] = (t & 1) ? bf_hi(u) : bf_lo(u);
        }
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
          if (i < nq) {
            const float4 p4 = *reinterpret_cast<const float4*>(&ss[i][r]);
            float v = fmaf(p4.x, vf[0], acc[i]);
            v = fmaf(p4.y, vf[1], v);
            v = fmaf(p4.z, vf[2], v);
            acc[i] = fmaf(p4.w, vf[3], v);
          }
        }
      }
      for (; r < nr; ++r) {
        const uint32_t u = sv[r][t >> 1];
        const float vf = (t & 1) ? bf_hi(u) : bf_lo(u);
#pragma unroll
        for (int i = 0; i < NQ; ++i)
          if (i < nq) acc[i] = fmaf(ss[i][r], vf, acc[i]);
      }
    }
  }
  __syncthreads();
  float* out = part + (((size_t)bh * p.groups + grp) * p.splits + split) * kGroup * kPart;
#pragma unroll
  for (int i = 0; i < NQ; ++i) {
    if (i >= nq) break;
    if (t == 0) {
      out[i * kPart] = sm_m[i];
      out[i * kPart + 1] = sm_l[i];
    }
    out[i * kPart + 2 + t] = acc[i];
  }
}

// One CTA per query. Thread t merges feature t of the splits' partials; every thread
// loads the splits' (max, sum) pairs too (the same addresses across the CTA, one
// transaction per warp), so that a batch of up to 32 splits is one round of
// independent loads and the merge needs no barrier. Batches are merged in split
// order, each rescaled to the running maximum.
__global__ void __launch_bounds__(kThreads)
decode_combine_kernel(const float* __restrict__ part, const float* __restrict__ ret,
                      const float* __restrict__ beta, __nv_bfloat16* __restrict__ out,
                      const DecodeParams p) {
  const int bh = blockIdx.x, t = threadIdx.x;
  const float bt = beta[bh % p.H];
  const float g = 1.f / (1.f + expf(-bt));
  const size_t sstride = (size_t)kGroup * kPart;
  for (int qi = blockIdx.y; qi < p.n; qi += gridDim.y) {
    const int grp = qi / kGroup, i = qi % kGroup;
    const float* pb = part + ((size_t)bh * p.groups + grp) * p.splits * kGroup * kPart + i * kPart;
    const float* rec = ret + ((size_t)bh * p.groups + grp) * kGroup * kRet + i * kRet;
    float m = -INFINITY, l = 0.f, a = 0.f;
    for (int s0 = 0; s0 < p.splits; s0 += 32) {
      float mx[32], sm[32], v[32];
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        mx[u] = -INFINITY;
        sm[u] = 0.f;
        v[u] = 0.f;
        if (s0 + u < p.splits) {
          const float* ps = pb + (size_t)(s0 + u) * sstride;
          mx[u] = ps[0];
          sm[u] = ps[1];
          v[u] = ps[2 + t];
        }
      }
      float mb = -INFINITY;
#pragma unroll
      for (int u = 0; u < 32; ++u) mb = fmaxf(mb, mx[u]);
      const float mn = fmaxf(m, mb);
      if (mn == -INFINITY) continue;  // no split of this batch (or before) saw a row
      const float sc = m == -INFINITY ? 0.f : exp2f(m - mn);
      l *= sc;
      a *= sc;
      // a split that saw none of the query's rows has max -inf and weight 0
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const float f = mx[u] == -INFINITY ? 0.f : exp2f(mx[u] - mn);
        l = fmaf(sm[u], f, l);
        a = fmaf(v[u], f, a);
      }
      m = mn;
    }
    const float den = rec[D];
    const float amem = den != 0.f ? rec[t] / den : 0.f;
    const float adot = a / l;
    out[((size_t)bh * p.n + qi) * D + t] = __float2bfloat16(g * amem + (1.f - g) * adot);
  }
}

// Cache split: one 64-row chunk per CTA while the splits and the retrieval CTA of
// every (head, group) fit one wave of four CTAs per SM, more chunks per CTA beyond;
// at most kMaxSplits splits.
void decode_splits(int BH, int n, int pos, int sms, int* splits, int* cps) {
  const int groups = (n + kGroup - 1) / kGroup;
  const int chunks = (pos + n + kRows - 1) / kRows;
  const long long want = 4LL * sms / ((long long)BH * groups) - kRetCTAs;
  int s = want < 1 ? 1 : (want > kMaxSplits ? kMaxSplits : (int)want);
  if (s > chunks) s = chunks;
  *cps = (chunks + s - 1) / s;
  *splits = (chunks + *cps - 1) / *cps;
}

}  // namespace

size_t bf16_decode_workspace_bytes(int BH, int n, int pos, int sms) {
  int splits = 0, cps = 0;
  decode_splits(BH, n, pos, sms, &splits, &cps);
  const int groups = (n + kGroup - 1) / kGroup;
  return ((size_t)BH * groups * splits * kGroup * kPart + (size_t)BH * groups * kGroup * kRet) *
         sizeof(float);
}

cudaError_t bf16_decode_launch(const __nv_bfloat16* q, const __nv_bfloat16* k,
                               const __nv_bfloat16* v, __nv_bfloat16* k_cache,
                               __nv_bfloat16* v_cache, const float* beta, const float* M,
                               const float* z, __nv_bfloat16* out, float* part, int BH, int H,
                               int n, int pos, int N, int sms, cudaStream_t stream) {
  DecodeParams p;
  p.n = n;
  p.pos = pos;
  p.N = N;
  p.H = H;
  p.groups = (n + kGroup - 1) / kGroup;
  decode_splits(BH, n, pos, sms, &p.splits, &p.chunks_per_split);
  const dim3 gp(p.splits + kRetCTAs, BH, p.groups), gc(BH, n < 65535 ? n : 65535);
  float* ret = part + (size_t)BH * p.groups * p.splits * kGroup * kPart;
  // the compiled width must hold the widest group: min(n, 16) queries
  const int w = n > 8 ? kGroup : n > 4 ? 8 : n > 2 ? 4 : n;
  switch (w) {
#define DECODE_CASE(W)                                                                      \
  case W:                                                                                   \
    decode_partial_kernel<W><<<gp, kThreads, 0, stream>>>(q, k, v, k_cache, v_cache, M, z,    \
                                                          part, ret, p);                    \
    decode_combine_kernel<<<gc, kThreads, 0, stream>>>(part, ret, beta, out, p);             \
    break;
    DECODE_CASE(1)
    DECODE_CASE(2)
    DECODE_CASE(4)
    DECODE_CASE(8)
    DECODE_CASE(16)
#undef DECODE_CASE
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace infini
