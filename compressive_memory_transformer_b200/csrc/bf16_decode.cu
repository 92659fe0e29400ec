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
//   decode_combine_kernel  grid (BH, query groups). Merges the splits' partials,
//                          adds the retrieval from the fp32 state (M read once per
//                          group, row-coalesced float4 loads spread over the four
//                          warps) and the gate, writes out in bf16.
// Both kernels are compiled for query-group widths 1, 2, 4, 8 and 16, so a single
// token carries no idle accumulators.
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

struct DecodeParams {
  int n, pos, N, H, splits, chunks_per_split, groups;
};

__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

template <int NQ>
__global__ void __launch_bounds__(kThreads)
decode_partial_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ knew,
                      const __nv_bfloat16* __restrict__ vnew, __nv_bfloat16* __restrict__ kc,
                      __nv_bfloat16* __restrict__ vc, float* __restrict__ part,
                      const DecodeParams p) {
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
    for (int e = t; e < nr * (D / 8); e += kThreads) {
      const int row = e / (D / 8), c = e % (D / 8);
      const int R = r0 + row;
      uint4 kk, vv;
      if (R < p.pos) {
        kk = *reinterpret_cast<const uint4*>(kc + base + (size_t)R * D + c * 8);
        vv = *reinterpret_cast<const uint4*>(vc + base + (size_t)R * D + c * 8);
      } else {
        const size_t src = ((size_t)bh * p.n + (R - p.pos)) * D + c * 8;
        kk = *reinterpret_cast<const uint4*>(knew + src);
        vv = *reinterpret_cast<const uint4*>(vnew + src);
        if (writer) {
          *reinterpret_cast<uint4*>(kc + base + (size_t)R * D + c * 8) = kk;
          *reinterpret_cast<uint4*>(vc + base + (size_t)R * D + c * 8) = vv;
        }
      }
      *reinterpret_cast<uint4*>(&sk[row][c * 4]) = kk;
      *reinterpret_cast<uint4*>(&sv[row][c * 4]) = vv;
    }
    __syncthreads();
    // scores: thread pair (2r, 2r + 1) covers row r, features [64h, 64h + 64); the
    // pair word read at step j is rotated by 2r + h, so a warp's 32 reads fall in 32
    // different banks
    {
      const int r = t >> 1, h = t & 1;
      float kf[64];
      if (r < nr) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const uint32_t u = sk[r][32 * h + ((j + 2 * r + h) & 31)];
          kf[2 * j] = bf_lo(u);
          kf[2 * j + 1] = bf_hi(u);
        }
      }
      for (int i = 0; i < nq; ++i) {
        float s = 0.f;
        if (r < nr) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int f = 64 * h + 2 * ((j + 2 * r + h) & 31);
            const float2 qf = *reinterpret_cast<const float2*>(&sq[i][f]);
            s = fmaf(qf.x, kf[2 * j], s);
            s = fmaf(qf.y, kf[2 * j + 1], s);
          }
        }
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        if (h == 0) ss[i][r] = (r < nr && r0 + r <= p.pos + q0 + i) ? s : -INFINITY;
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
#pragma unroll 4
      for (int r = 0; r < nr; ++r) {
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

template <int NQ>
__global__ void __launch_bounds__(kThreads)
decode_combine_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ part,
                      const float* __restrict__ beta, const float* __restrict__ M,
                      const float* __restrict__ z, __nv_bfloat16* __restrict__ out,
                      const DecodeParams p) {
  __shared__ float sphi[NQ][D];  // sigma(q)
  __shared__ float sden[NQ][kThreads / 32];
  __shared__ __align__(16) float sr[kThreads / 32][NQ][D];  // per-warp partial retrievals
  const int bh = blockIdx.x, grp = blockIdx.y, t = threadIdx.x, lane = t & 31, w = t >> 5;
  const int q0 = grp * kGroup;
  const int nq = min(NQ, p.n - q0);
  const float zt = z[(size_t)bh * D + t];
  for (int i = 0; i < nq; ++i) {
    const float phi = elu1(__bfloat162float(q[((size_t)bh * p.n + q0 + i) * D + t]));
    sphi[i][t] = phi;
    float dp = phi * zt;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dp += __shfl_xor_sync(0xffffffffu, dp, o);
    if (lane == 0) sden[i][w] = dp;
  }
  __syncthreads();
  // retrieval R[i][c] = sum_k sigma(q_i)[k] M[k][c]: warp w takes rows k = w, w + 4, ...,
  // lane takes columns [4 lane, 4 lane + 4) (one 512-byte row per warp load), eight
  // rows in flight per thread
  {
    float4 rr[NQ];
#pragma unroll
    for (int i = 0; i < NQ; ++i) rr[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    const float4* Mb = reinterpret_cast<const float4*>(M + (size_t)bh * D * D);
#pragma unroll 8
    for (int k = w; k < D; k += kThreads / 32) {
      const float4 m = Mb[(size_t)k * (D / 4) + lane];
#pragma unroll
      for (int i = 0; i < NQ; ++i) {
        if (i < nq) {
          const float ph = sphi[i][k];
          rr[i].x = fmaf(ph, m.x, rr[i].x);
          rr[i].y = fmaf(ph, m.y, rr[i].y);
          rr[i].z = fmaf(ph, m.z, rr[i].z);
          rr[i].w = fmaf(ph, m.w, rr[i].w);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < NQ; ++i)
      if (i < nq) *reinterpret_cast<float4*>(&sr[w][i][4 * lane]) = rr[i];
  }
  __syncthreads();
  const float bt = beta[bh % p.H];
  const float g = 1.f / (1.f + expf(-bt));
  const float* pb = part + ((size_t)bh * p.groups + grp) * p.splits * kGroup * kPart;
  for (int i = 0; i < nq; ++i) {
    float m = -INFINITY;
    for (int s = 0; s < p.splits; ++s) m = fmaxf(m, pb[(s * kGroup + i) * kPart]);
    float l = 0.f, a = 0.f;
    for (int s = 0; s < p.splits; ++s) {
      const float* ps = pb + (s * kGroup + i) * kPart;
      if (ps[0] == -INFINITY) continue;  // this split saw none of the query's rows
      const float f = exp2f(ps[0] - m);
      l = fmaf(ps[1], f, l);
      a = fmaf(ps[2 + t], f, a);
    }
    const float den = (sden[i][0] + sden[i][1]) + (sden[i][2] + sden[i][3]);
    const float r = (sr[0][i][t] + sr[1][i][t]) + (sr[2][i][t] + sr[3][i][t]);
    const float amem = den != 0.f ? r / den : 0.f;
    const float adot = a / l;
    out[((size_t)bh * p.n + q0 + i) * D + t] = __float2bfloat16(g * amem + (1.f - g) * adot);
  }
}

}  // namespace

size_t bf16_decode_workspace_bytes(int BH, int n, int pos, int sms) {
  const int groups = (n + kGroup - 1) / kGroup;
  const int chunks = (pos + n + kRows - 1) / kRows;
  const int want = (2 * sms + BH * groups - 1) / (BH * groups);
  int splits = want < 1 ? 1 : want;
  if (splits > chunks) splits = chunks;
  const int cps = (chunks + splits - 1) / splits;
  splits = (chunks + cps - 1) / cps;
  return (size_t)BH * groups * splits * kGroup * kPart * sizeof(float);
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
  const int chunks = (pos + n + kRows - 1) / kRows;
  const int want = (2 * sms + BH * p.groups - 1) / (BH * p.groups);
  int splits = want < 1 ? 1 : want;
  if (splits > chunks) splits = chunks;
  p.chunks_per_split = (chunks + splits - 1) / splits;
  p.splits = (chunks + p.chunks_per_split - 1) / p.chunks_per_split;
  const dim3 gp(p.splits, BH, p.groups), gc(BH, p.groups);
  // the compiled width must hold the widest group: min(n, 16) queries
  const int w = n > 8 ? kGroup : n > 4 ? 8 : n > 2 ? 4 : n;
  switch (w) {
#define DECODE_CASE(W)                                                                      \
  case W:                                                                                   \
    decode_partial_kernel<W><<<gp, kThreads, 0, stream>>>(q, k, v, k_cache, v_cache, part, p); \
    decode_combine_kernel<W><<<gc, kThreads, 0, stream>>>(q, part, beta, M, z, out, p);      \
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
