// f32_path.cu — fp32 Infini-attention forward on CUDA cores (SIMT).
//
// Correctness path for fp32 inputs (any head width 1 <= d <= 128, any segment
// length): all arithmetic in fp32 FMA, no tensor cores, so the result stays
// within about 1e-6 of the exact value. Two kernels per call:
//   f32_state_kernel : per (batch*head, 32-column block of M), walks the segments
//                      in order, emits the state each segment reads (M_{s-1},
//                      z_{s-1}) and applies the Linear or Linear+Delta update.
//   f32_attn_kernel  : one warp per query row: causal softmax attention inside
//                      the segment (online max/sum), retrieval from the emitted
//                      state, gate.
// Equations: "Leave No Context Behind" (arXiv 2404.07143) as quoted on
// llm-papers-study.pages.dev, sections 3.1 (A_dot), 3.3 (A_mem), 3.4 (updates),
// 3.5 (gate).
#include <cuda_runtime.h>
#include <cmath>
#include <cstdint>

#include "f32_path.h"

namespace infini {
namespace {

constexpr int kCB = 32;      // columns of M per state block
constexpr int kTC = 32;      // tokens per state chunk
constexpr int kMaxD = 128;
constexpr int kStateThreads = 256;

__device__ __forceinline__ float elu1_precise(float x) { return x > 0.f ? x + 1.f : expf(x); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// grid: (B*H, ceil(d/32)); block: 256 threads.
// Writes Mprev[bh][s] (columns of this block) and, from block 0, zprev[bh][s]
// for s = 0..S-1, plus zprev[bh][S] = final z; M_out for this block's columns.
__global__ void __launch_bounds__(kStateThreads)
f32_state_kernel(const float* __restrict__ k, const float* __restrict__ v,
                 const float* __restrict__ M_in, const float* __restrict__ z_in,
                 float* __restrict__ M_out, float* __restrict__ Mprev,
                 float* __restrict__ zprev, long long L, int N, int d, int S, int mode) {
  __shared__ float sM[kMaxD][kCB];     // M_{s-1}, this block's columns
  __shared__ float sPhi[kTC][kMaxD];   // sigma(K) of the token chunk
  __shared__ float sU[kTC][kCB];       // V (Linear) or V - R (Delta), block columns
  __shared__ float sDen[kTC];
  __shared__ float sZ[kMaxD];

  const int bh = blockIdx.x;
  const int c0 = blockIdx.y * kCB;
  const int nc = min(kCB, d - c0);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const size_t dd = (size_t)d * d;
  const float* kh = k + (size_t)bh * L * d;
  const float* vh = v + (size_t)bh * L * d;

  for (int i = tid; i < d; i += kStateThreads) sZ[i] = z_in ? z_in[(size_t)bh * d + i] : 0.f;
  for (int e = tid; e < d * kCB; e += kStateThreads) {
    const int r = e / kCB, c = e % kCB;
    sM[r][c] = (M_in && c < nc) ? M_in[(size_t)bh * dd + (size_t)r * d + c0 + c] : 0.f;
  }
  __syncthreads();

  constexpr int kPer = kMaxD * kCB / kStateThreads;  // 16 state elements per thread
  for (int s = 0; s < S; ++s) {
    const long long t0 = (long long)s * N;
    const int n = (int)min((long long)N, L - t0);
    float* mp = Mprev + ((size_t)bh * S + s) * dd;
    for (int e = tid; e < d * kCB; e += kStateThreads) {
      const int r = e / kCB, c = e % kCB;
      if (c < nc) mp[(size_t)r * d + c0 + c] = sM[r][c];
    }
    if (blockIdx.y == 0)
      for (int i = tid; i < d; i += kStateThreads) zprev[((size_t)bh * (S + 1) + s) * d + i] = sZ[i];

    float dM[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) dM[i] = 0.f;
    float dz = 0.f;  // threads tid < d accumulate z for feature tid

    for (int tc = 0; tc < n; tc += kTC) {
      const int tn = min(kTC, n - tc);
      for (int e = tid; e < kTC * d; e += kStateThreads) {
        const int t = e / d, c = e % d;
        sPhi[t][c] = t < tn ? elu1_precise(kh[(size_t)(t0 + tc + t) * d + c]) : 0.f;
      }
      for (int e = tid; e < kTC * kCB; e += kStateThreads) {
        const int t = e / kCB, c = e % kCB;
        sU[t][c] = (t < tn && c < nc) ? vh[(size_t)(t0 + tc + t) * d + c0 + c] : 0.f;
      }
      __syncthreads();
      if (mode == 1) {
        for (int t = warp; t < kTC; t += kStateThreads / 32) {
          float acc = 0.f;
          for (int c = lane; c < d; c += 32) acc = fmaf(sPhi[t][c], sZ[c], acc);
          acc = warp_sum(acc);
          if (lane == 0) sDen[t] = acc;
        }
        __syncthreads();
        // U = V - sigma(K) M_{s-1} / (sigma(K) z_{s-1}); rows with den == 0 keep V
        float u[kTC * kCB / kStateThreads];
#pragma unroll
        for (int i = 0; i < kTC * kCB / kStateThreads; ++i) {
          const int e = tid + i * kStateThreads;
          const int t = e / kCB, c = e % kCB;
          float num = 0.f;
          for (int r = 0; r < d; ++r) num = fmaf(sPhi[t][r], sM[r][c], num);
          const float den = sDen[t];
          u[i] = sU[t][c] - (den != 0.f ? num / den : 0.f);
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < kTC * kCB / kStateThreads; ++i) {
          const int e = tid + i * kStateThreads;
          sU[e / kCB][e % kCB] = u[i];
        }
        __syncthreads();
      }
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int e = tid + i * kStateThreads;
        const int r = e / kCB, c = e % kCB;
        if (r < d) {
          float acc = dM[i];
          for (int t = 0; t < tn; ++t) acc = fmaf(sPhi[t][r], sU[t][c], acc);
          dM[i] = acc;
        }
      }
      if (tid < d)
        for (int t = 0; t < tn; ++t) dz += sPhi[t][tid];
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = tid + i * kStateThreads;
      const int r = e / kCB, c = e % kCB;
      if (r < d) sM[r][c] += dM[i];
    }
    if (tid < d) sZ[tid] += dz;
    __syncthreads();
  }
  if (M_out)
    for (int e = tid; e < d * kCB; e += kStateThreads) {
      const int r = e / kCB, c = e % kCB;
      if (c < nc) M_out[(size_t)bh * dd + (size_t)r * d + c0 + c] = sM[r][c];
    }
  if (blockIdx.y == 0)
    for (int i = tid; i < d; i += kStateThreads) zprev[((size_t)bh * (S + 1) + S) * d + i] = sZ[i];
}

constexpr int kAttnWarps = 8;

// grid: (ceil(L / 8), B*H); one warp per query row.
__global__ void __launch_bounds__(kAttnWarps * 32)
f32_attn_kernel(const float* __restrict__ q, const float* __restrict__ k,
                const float* __restrict__ v, const float* __restrict__ beta,
                const float* __restrict__ Mprev, const float* __restrict__ zprev,
                float* __restrict__ out, float* __restrict__ z_out, long long L, int N, int d,
                int H, int S) {
  const int bh = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kAttnWarps + (threadIdx.x >> 5);

  if (z_out && blockIdx.x == 0)
    for (int i = threadIdx.x; i < d; i += blockDim.x)
      z_out[(size_t)bh * d + i] = zprev[((size_t)bh * (S + 1) + S) * d + i];
  if (row >= L) return;

  const int s = (int)(row / N);
  const long long s0 = (long long)s * N;
  const size_t hoff = (size_t)bh * L * d;
  const float* qr = q + hoff + (size_t)row * d;
  constexpr int U = kMaxD / 32;
  float qv[U], o[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int c = lane + 32 * u;
    qv[u] = c < d ? qr[c] : 0.f;
    o[u] = 0.f;
  }
  const float scale = 1.0f / sqrtf((float)d);
  float m = -INFINITY, l = 0.f;
  for (long long j = s0; j <= row; ++j) {
    const float* kr = k + hoff + (size_t)j * d;
    const float* vr = v + hoff + (size_t)j * d;
    float part = 0.f;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = lane + 32 * u;
      if (c < d) part = fmaf(qv[u], kr[c], part);
    }
    const float sc = warp_sum(part) * scale;
    const float m_new = fmaxf(m, sc);
    const float corr = expf(m - m_new);  // 0 on the first key (m = -inf)
    const float p = expf(sc - m_new);
    l = l * corr + p;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = lane + 32 * u;
      o[u] = o[u] * corr + (c < d ? p * vr[c] : 0.f);
    }
    m = m_new;
  }
  // retrieval with the state before this segment's update
  const float* Mp = Mprev + ((size_t)bh * S + s) * (size_t)d * d;
  const float* zp = zprev + ((size_t)bh * (S + 1) + s) * d;
  float phi[U];
  float den_part = 0.f;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int c = lane + 32 * u;
    phi[u] = c < d ? elu1_precise(qv[u]) : 0.f;
    if (c < d) den_part = fmaf(phi[u], zp[c], den_part);
  }
  const float den = warp_sum(den_part);
  float num[U];
#pragma unroll
  for (int u = 0; u < U; ++u) num[u] = 0.f;
#pragma unroll
  for (int ur = 0; ur < U; ++ur) {
    for (int rr = 0; rr < 32; ++rr) {
      const int r = 32 * ur + rr;
      if (r >= d) break;
      const float pr = __shfl_sync(0xffffffffu, phi[ur], rr);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = lane + 32 * u;
        if (c < d) num[u] = fmaf(pr, Mp[(size_t)r * d + c], num[u]);
      }
    }
  }
  const float b = beta[bh % H];
  const float g = 1.f / (1.f + expf(-b));
  float* orow = out + hoff + (size_t)row * d;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int c = lane + 32 * u;
    if (c < d) {
      const float a_mem = den != 0.f ? num[u] / den : 0.f;
      orow[c] = g * a_mem + (1.f - g) * (o[u] / l);
    }
  }
}

}  // namespace

size_t f32_workspace_bytes(int BH, int S, int d) {
  const size_t mp = (size_t)BH * S * d * d * sizeof(float);
  const size_t zp = (size_t)BH * (S + 1) * d * sizeof(float);
  return ((mp + 255) & ~(size_t)255) + ((zp + 255) & ~(size_t)255);
}

cudaError_t f32_forward_launch(const float* q, const float* k, const float* v, const float* beta,
                               const float* M_in, const float* z_in, float* out, float* M_out,
                               float* z_out, int BH, int H, long long L, int N, int d, int mode,
                               void* workspace, cudaStream_t stream) {
  const int S = (int)((L + N - 1) / N);
  const size_t mp = (size_t)BH * S * d * d * sizeof(float);
  float* Mprev = static_cast<float*>(workspace);
  float* zprev = reinterpret_cast<float*>(static_cast<char*>(workspace) + ((mp + 255) & ~(size_t)255));
  dim3 g1(BH, (d + kCB - 1) / kCB);
  f32_state_kernel<<<g1, kStateThreads, 0, stream>>>(k, v, M_in, z_in, M_out, Mprev, zprev, L, N,
                                                     d, S, mode);
  dim3 g2((unsigned)((L + kAttnWarps - 1) / kAttnWarps), BH);
  f32_attn_kernel<<<g2, kAttnWarps * 32, 0, stream>>>(q, k, v, beta, Mprev, zprev, out, z_out, L,
                                                      N, d, H, S);
  return cudaGetLastError();
}

}  // namespace infini
