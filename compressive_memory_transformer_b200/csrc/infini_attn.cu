// infini_attn.cu — the C ABI (include/infini_attn.h): argument checks, scratch
// memory, and the launch sequence of the forward.
//
// bf16 (d = 128), several segments:
//   Linear+Delta: zpart -> zscan -> state (tcgen05 bf16, sigma(K) as a hi/lo pair)
//                 -> chain (G_s M_{s-1} on tcgen05 tf32) -> attn (tcgen05 bf16)
//   Linear:       state (also the sums of sigma(K)) -> chain (with the z scan) -> attn
// one segment (every step call): prep_first, then the one-segment update (a second
//   stream) beside attn
// fp32 (d <= 128): f32_state -> f32_attn (CUDA cores)
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "infini_attn.h"
#include "bf16_path.h"
#include "f32_path.h"
#include "sm100.cuh"

namespace infini {

__device__ int g_device_error = 0;
__device__ unsigned long long g_wait_timeout_ns = 4000000000ull;  // 4 s per wait

cudaError_t bf16_state_set_attributes();
cudaError_t bf16_attn_set_attributes();
cudaError_t bf16_bwd_set_attributes();
cudaError_t bf16_gemm_set_attributes();
cudaError_t bf16_step_state_set_attributes();

namespace {

constexpr int kMaxDevices = 64;
std::atomic<int> g_prepared[kMaxDevices];
std::mutex g_prepare_mu;

// A second stream of each device, for one-segment calls: the state update runs on
// it beside the attention kernel, forked from and joined back into the caller's
// stream inside the call. The mutex keeps each fork..join sequence whole when
// several host threads call at once.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  std::mutex mu;
};
SideStream g_side[kMaxDevices];

cudaError_t prepare_device(int* dev_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  *dev_out = dev;
  if (g_prepared[dev].load(std::memory_order_acquire)) return cudaSuccess;
  std::lock_guard<std::mutex> lk(g_prepare_mu);
  if (g_prepared[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = bf16_state_set_attributes();
  if (e == cudaSuccess) e = bf16_attn_set_attributes();
  if (e == cudaSuccess) e = bf16_bwd_set_attributes();
  if (e == cudaSuccess) e = bf16_gemm_set_attributes();
  if (e == cudaSuccess) e = bf16_step_state_set_attributes();
  SideStream& sd = g_side[dev];
  if (e == cudaSuccess && !sd.stream) e = cudaStreamCreateWithFlags(&sd.stream, cudaStreamNonBlocking);
  if (e == cudaSuccess && !sd.fork) e = cudaEventCreateWithFlags(&sd.fork, cudaEventDisableTiming);
  if (e == cudaSuccess && !sd.join) e = cudaEventCreateWithFlags(&sd.join, cudaEventDisableTiming);
  if (e == cudaSuccess) g_prepared[dev].store(1, std::memory_order_release);
  return e;
}

// Copies (or zero-fills) the state when there is nothing to process.
__global__ void pass_state_kernel(const float* M_in, const float* z_in, float* M_out,
                                  float* z_out, long long nM, long long nz) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < nM;
       i += (long long)gridDim.x * blockDim.x) {
    if (i < nz && z_out) z_out[i] = z_in ? z_in[i] : 0.f;
    if (M_out) M_out[i] = M_in ? M_in[i] : 0.f;
  }
}

// (M_out, z_out) = (M_in, z_in) (or zero) + the sum of `count` state blocks, added in
// block order (the Linear memory is a plain sum over segments, section 3.4).
__global__ void state_sum_kernel(const float* dM, const float* dz, int count, const float* M_in,
                                 const float* z_in, float* M_out, float* z_out, long long nM,
                                 long long nz) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < nM;
       i += (long long)gridDim.x * blockDim.x) {
    float m = M_in ? M_in[i] : 0.f;
    for (int c = 0; c < count; ++c) m += dM[(long long)c * nM + i];
    M_out[i] = m;
    if (i < nz) {
      float zz = z_in ? z_in[i] : 0.f;
      for (int c = 0; c < count; ++c) zz += dz[(long long)c * nz + i];
      z_out[i] = zz;
    }
  }
}

__global__ void timeout_selftest_kernel(unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives on this barrier: the wait must run out and report
    const uint32_t a = smem_u32(&bar);
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(a, 0)) {
      if (globaltimer_ns() - t0 > timeout_ns) {
        raise_device_error(kDevErrTimeout);
        break;
      }
    }
  }
}

bool overflows(long long a, long long b) { return a != 0 && b > (long long)(INT64_MAX / a); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

int check_common(const void* q, const void* k, const void* v, const float* beta,
                 const float* M_in, const float* z_in, const void* out, const float* M_out,
                 const float* z_out, int B, int H, long long L, int N, int d, int mode,
                 size_t esize, int H_kv = 0) {
  if (H_kv == 0) H_kv = H;
  if (!beta) return INFINI_ERR_NULL;
  if (L > 0 && (!q || !k || !v || !out)) return INFINI_ERR_NULL;
  if ((M_in == nullptr) != (z_in == nullptr)) return INFINI_ERR_NULL;
  if ((M_out == nullptr) != (z_out == nullptr)) return INFINI_ERR_NULL;
  if (B < 1 || H < 1 || N < 1 || L < 0 || d < 1) return INFINI_ERR_SHAPE;
  if (mode != INFINI_LINEAR && mode != INFINI_DELTA) return INFINI_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  if (BH > (1LL << 30)) return INFINI_ERR_SHAPE;
  if (overflows(BH, L) || overflows(BH * L, d) || overflows(BH * L * d, (long long)esize))
    return INFINI_ERR_SHAPE;
  if (L >= (1LL << 31)) return INFINI_ERR_SHAPE;
  if (H_kv < 1 || H % H_kv != 0) return INFINI_ERR_SHAPE;
  const long long BHkv = (long long)B * H_kv;
  const size_t nio = (size_t)(BH * L * d) * esize, nkv = (size_t)(BHkv * L * d) * esize;
  const size_t nM = (size_t)BHkv * d * d * sizeof(float), nz = (size_t)BHkv * d * sizeof(float);
  if (overlap(out, nio, q, nio) || overlap(out, nio, k, nkv) || overlap(out, nio, v, nkv) ||
      overlap(out, nio, M_in, nM) || overlap(out, nio, z_in, nz) ||
      overlap(out, nio, M_out, nM) || overlap(out, nio, z_out, nz))
    return INFINI_ERR_ALIAS;
  return INFINI_OK;
}

int pass_state(const float* M_in, const float* z_in, float* M_out, float* z_out, long long BH,
               int d, cudaStream_t stream) {
  if (!M_out) return INFINI_OK;
  const long long nM = BH * d * d, nz = BH * d;
  pass_state_kernel<<<(unsigned)min((nM + 255) / 256, 4096LL), 256, 0, stream>>>(M_in, z_in,
                                                                                  M_out, z_out,
                                                                                  nM, nz);
  return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

struct Scratch {
  void* ptr = nullptr;
  bool owned = false;
  cudaStream_t stream = nullptr;
  ~Scratch() {
    if (owned && ptr) cudaFreeAsync(ptr, stream);
  }
};

int get_scratch(Scratch& s, size_t bytes, const infini_attn_opts_t* opts, cudaStream_t stream) {
  if (bytes == 0) return INFINI_OK;
  if (opts && opts->workspace) {
    if (opts->workspace_bytes < bytes) return INFINI_ERR_NOMEM;
    if ((reinterpret_cast<uintptr_t>(opts->workspace) & 255u) != 0) return INFINI_ERR_ALIGN;
    s.ptr = opts->workspace;
    return INFINI_OK;
  }
  if (cudaMallocAsync(&s.ptr, bytes, stream) != cudaSuccess) {
    cudaGetLastError();
    s.ptr = nullptr;
    return INFINI_ERR_NOMEM;
  }
  s.owned = true;
  s.stream = stream;
  return INFINI_OK;
}

int device_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  return sms;
}

// Scratch of one bf16 forward: the state path's workspace, then (one segment) the
// one-segment update's partial sums, then (calls with fewer query-tile pairs than
// SMs) the attention's split scratch.
struct FwdPlan {
  int CH = 1, CL = 1;        // multi-segment state GEMM: token chunks
  int sCH = 0, sCL = 0;      // one segment: token chunks of the update
  Bf16AttnSplit split;
  size_t state_bytes = 0, step_bytes = 0, bytes = 0;
};

FwdPlan fwd_plan(int BH, int BHkv, int S, int N, long long L) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  FwdPlan f;
  f.CL = N;
  bf16_state_plan(BHkv, S, N, &f.CH, &f.CL);
  f.split = bf16_attn_split_plan(BH, S, N, L, device_sms());
  f.state_bytes = up(bf16_workspace_bytes(BHkv, S, f.CH));
  if (S == 1 && L > 0) {
    bf16_step_state_plan(BHkv, (int)min((long long)N, L), &f.sCH, &f.sCL);
    f.step_bytes = up(bf16_step_state_bytes(BHkv, f.sCH));
  }
  f.bytes = f.state_bytes + f.step_bytes + bf16_attn_split_bytes(f.split, BH, S, N, L);
  return f;
}

void record(const infini_attn_opts_t* opts, int i, cudaStream_t stream) {
  if (opts && opts->stage_events[i])
    cudaEventRecord(static_cast<cudaEvent_t>(opts->stage_events[i]), stream);
}

int forward_impl(const void* q, const void* k, const void* v, const float* beta,
                 const float* M_in, const float* z_in, void* out, float* M_out, float* z_out,
                 int B, int H, long long L, int N, int d, int mode, int dtype,
                 const infini_attn_opts_t* opts, cudaStream_t stream, int H_kv = 0,
                 int layout = INFINI_LAYOUT_BHLD) {
  if (dtype != INFINI_DTYPE_BF16 && dtype != INFINI_DTYPE_F32) return INFINI_ERR_UNSUPPORTED;
  if (H_kv == 0) H_kv = H;
  // the fp32 path's attention grid has a row per head
  if (dtype == INFINI_DTYPE_F32 && (long long)B * H > 65535) return INFINI_ERR_SHAPE;
  const size_t esize = dtype == INFINI_DTYPE_BF16 ? 2 : 4;
  int st = check_common(q, k, v, beta, M_in, z_in, out, M_out, z_out, B, H, L, N, d, mode, esize,
                        H_kv);
  if (st != INFINI_OK) return st;
  if (layout != INFINI_LAYOUT_BHLD && layout != INFINI_LAYOUT_BLHD) return INFINI_ERR_UNSUPPORTED;
  if (dtype == INFINI_DTYPE_F32 && (layout != INFINI_LAYOUT_BHLD || H_kv != H))
    return INFINI_ERR_UNSUPPORTED;
  if (dtype == INFINI_DTYPE_BF16 && d != 128) return INFINI_ERR_UNSUPPORTED;
  if (dtype == INFINI_DTYPE_F32 && d > 128) return INFINI_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return INFINI_ERR_ALIGN;
  if ((M_in && !aligned16(M_in)) || (M_out && !aligned16(M_out))) return INFINI_ERR_ALIGN;
  const int BH = B * H, BHkv = B * H_kv;
  const Bf16Layout lay = layout == INFINI_LAYOUT_BLHD ? Bf16Layout::blhd(B, H, H_kv, L)
                                                      : Bf16Layout{B, H, H_kv, (long long)H * L * d,
                                                                   L * d, d, (long long)H_kv * L * d,
                                                                   L * d, d};
  if (L == 0) {
    record(opts, 0, stream);
    st = pass_state(M_in, z_in, M_out, z_out, BHkv, d, stream);
    record(opts, 1, stream);
    record(opts, 2, stream);
    return st;
  }
  int dev = 0;
  if (prepare_device(&dev) != cudaSuccess) return INFINI_ERR_CUDA;
  const int S = (int)((L + N - 1) / N);
  if (dtype == INFINI_DTYPE_F32) {
    Scratch sc;
    st = get_scratch(sc, f32_workspace_bytes(BH, S, d), opts, stream);
    if (st != INFINI_OK) return st;
    record(opts, 0, stream);
    const cudaError_t e = f32_forward_launch(
        static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
        beta, M_in, z_in, static_cast<float*>(out), M_out, z_out, BH, H, L, N, d, mode, sc.ptr,
        stream);
    record(opts, 1, stream);
    record(opts, 2, stream);
    return e == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
  }
  const FwdPlan fp = fwd_plan(BH, BHkv, S, N, L);
  const int CH = fp.CH, CL = fp.CL;
  if ((long long)BHkv * S * CH >= (1LL << 31)) return INFINI_ERR_SHAPE;
  Scratch sc;
  st = get_scratch(sc, fp.bytes, opts, stream);
  if (st != INFINI_OK) return st;
  const Bf16Workspace ws = bf16_workspace_carve(sc.ptr, BHkv, S, CH);
  void* step_ws = fp.step_bytes ? static_cast<char*>(sc.ptr) + fp.state_bytes : nullptr;
  void* split_ws =
      fp.split.C ? static_cast<char*>(sc.ptr) + fp.state_bytes + fp.step_bytes : nullptr;
  const auto* qb = static_cast<const __nv_bfloat16*>(q);
  const auto* kb = static_cast<const __nv_bfloat16*>(k);
  const auto* vb = static_cast<const __nv_bfloat16*>(v);
  record(opts, 0, stream);
  if (S == 1) {
    // One segment: the attention reads only the incoming state (M_in, z_in), so it
    // runs beside the state update, which goes to the side stream and is joined
    // back before the call returns. The update is the one-segment kernel (chunks of
    // tokens in parallel, no chain); without M_out there is no update to make.
    const int nseg = (int)min((long long)N, L);
    unsigned* sctr = step_ws ? bf16_step_state_counters(step_ws, BHkv, fp.sCH) : nullptr;
    cudaError_t e = bf16_prep_first(M_in, z_in, ws, BHkv, S, stream, sctr, sctr ? 2 * BHkv : 0);
    if (e != cudaSuccess) return INFINI_ERR_CUDA;
    if (!M_out) {
      record(opts, 1, stream);
      e = bf16_attn_launch(qb, kb, vb, beta, static_cast<__nv_bfloat16*>(out), ws, BH, H, L, N,
                           S, stream, &lay, &fp.split, split_ws);
      record(opts, 2, stream);
      return e == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
    }
    SideStream& sd = g_side[dev];
    std::lock_guard<std::mutex> lk(sd.mu);
    e = cudaEventRecord(sd.fork, stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(sd.stream, sd.fork, 0);
    if (e != cudaSuccess) return INFINI_ERR_CUDA;
    const cudaError_t es = bf16_step_state_launch(kb, vb, M_in, M_out, z_out, ws, step_ws, BHkv,
                                                  nseg, fp.sCH, fp.sCL, mode, sd.stream, &lay);
    record(opts, 1, stream);
    // Beside the state update the attention keeps its tile pairs: split units would
    // want the SMs the update holds (measured on 8 heads of one 2048-token segment:
    // 33.6 us per step with pairs, 36.9 with whole tiles taken from the counter).
    const cudaError_t ea = bf16_attn_launch(qb, kb, vb, beta, static_cast<__nv_bfloat16*>(out),
                                            ws, BH, H, L, N, S, stream, &lay);
    // joined even after a launch error, so that the side stream never runs ahead of
    // the caller's stream
    cudaError_t ej = cudaEventRecord(sd.join, sd.stream);
    if (ej == cudaSuccess) ej = cudaStreamWaitEvent(stream, sd.join, 0);
    record(opts, 2, stream);
    return es == cudaSuccess && ea == cudaSuccess && ej == cudaSuccess ? INFINI_OK
                                                                        : INFINI_ERR_CUDA;
  }
  cudaError_t e = bf16_state_launch(kb, vb, M_in, z_in, M_out, z_out, ws, BHkv, L, N, S, CH, CL,
                                    mode, 0, stream, &lay);
  if (e != cudaSuccess) return INFINI_ERR_CUDA;
  record(opts, 1, stream);
  e = bf16_attn_launch(qb, kb, vb, beta, static_cast<__nv_bfloat16*>(out), ws, BH, H, L, N, S,
                       stream, &lay, &fp.split, split_ws);
  record(opts, 2, stream);
  return e == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

// The state path alone: (M_out, z_out) after L tokens (segments of N) from (M_in,
// z_in), without the attention outputs.
int state_update_impl(const void* k, const void* v, const float* M_in, const float* z_in,
                      float* M_out, float* z_out, int B, int H, long long L, int N, int d,
                      int mode, cudaStream_t stream) {
  if (!M_out || !z_out) return INFINI_ERR_NULL;
  if (L > 0 && (!k || !v)) return INFINI_ERR_NULL;
  if ((M_in == nullptr) != (z_in == nullptr)) return INFINI_ERR_NULL;
  if (B < 1 || H < 1 || N < 1 || L < 0 || d < 1) return INFINI_ERR_SHAPE;
  if (mode != INFINI_LINEAR && mode != INFINI_DELTA) return INFINI_ERR_UNSUPPORTED;
  if (d != 128) return INFINI_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  if (BH > (1LL << 30) || overflows(BH, L) || overflows(BH * L, (long long)d * 2) ||
      L >= (1LL << 31))
    return INFINI_ERR_SHAPE;
  if ((L > 0 && (!aligned16(k) || !aligned16(v))) || (M_in && !aligned16(M_in)) ||
      !aligned16(M_out))
    return INFINI_ERR_ALIGN;
  const size_t nio = (size_t)(BH * L * d) * 2;
  const size_t nM = (size_t)BH * d * d * sizeof(float), nz = (size_t)BH * d * sizeof(float);
  if (overlap(M_out, nM, k, nio) || overlap(M_out, nM, v, nio) || overlap(z_out, nz, k, nio) ||
      overlap(z_out, nz, v, nio) || overlap(M_out, nM, z_out, nz))
    return INFINI_ERR_ALIAS;
  if (L == 0) return pass_state(M_in, z_in, M_out, z_out, BH, d, stream);
  int dev = 0;
  if (prepare_device(&dev) != cudaSuccess) return INFINI_ERR_CUDA;
  const int S = (int)((L + N - 1) / N);
  int CH = 1, CL = N;
  bf16_state_plan((int)BH, S, N, &CH, &CL);
  if (BH * S * CH >= (1LL << 31)) return INFINI_ERR_SHAPE;
  Scratch sc;
  const int st = get_scratch(sc, bf16_workspace_bytes((int)BH, S, CH), nullptr, stream);
  if (st != INFINI_OK) return st;
  const Bf16Workspace ws = bf16_workspace_carve(sc.ptr, (int)BH, S, CH);
  const cudaError_t e = bf16_state_launch(static_cast<const __nv_bfloat16*>(k),
                                          static_cast<const __nv_bfloat16*>(v), M_in, z_in, M_out,
                                          z_out, ws, (int)BH, L, N, S, CH, CL, mode, 0, stream);
  return e == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

// Token-level decode: attention + retrieval + gate for the new tokens against the
// cache and the state as it stands (the new rows are also written into the caches),
// then, when the segment is complete, the segment's state update in place (the same
// calls as a one-segment step with M_out == M_in).
int decode_impl(const void* q, const void* k, const void* v, const float* beta, void* k_cache,
                void* v_cache, float* M, float* z, void* out, int B, int H, int n, int pos,
                int N, int d, int mode, cudaStream_t stream) {
  if (!q || !k || !v || !beta || !k_cache || !v_cache || !M || !z || !out) return INFINI_ERR_NULL;
  if (B < 1 || H < 1 || n < 1 || pos < 0 || N < 1 || (long long)pos + n > N)
    return INFINI_ERR_SHAPE;
  if (mode != INFINI_LINEAR && mode != INFINI_DELTA) return INFINI_ERR_UNSUPPORTED;
  if (d != 128) return INFINI_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  if (BH > (1LL << 30) || overflows(BH, (long long)N * d * 2)) return INFINI_ERR_SHAPE;
  // the decode grid has a row per head and a layer per group of 16 new tokens
  if (BH > 65535 || (n + 15) / 16 > 65535) return INFINI_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(k_cache) ||
      !aligned16(v_cache) || !aligned16(M) || !aligned16(z))
    return INFINI_ERR_ALIGN;
  const size_t nio = (size_t)(BH * n * d) * 2, ncache = (size_t)(BH * N * d) * 2;
  const size_t nM = (size_t)BH * d * d * sizeof(float), nz = (size_t)BH * d * sizeof(float);
  const void* ins[] = {q, k, v};
  for (const void* x : ins)
    if (overlap(out, nio, x, nio) || overlap(k_cache, ncache, x, nio) ||
        overlap(v_cache, ncache, x, nio))
      return INFINI_ERR_ALIAS;
  if (overlap(out, nio, k_cache, ncache) || overlap(out, nio, v_cache, ncache) ||
      overlap(out, nio, M, nM) || overlap(out, nio, z, nz) ||
      overlap(k_cache, ncache, v_cache, ncache) || overlap(k_cache, ncache, M, nM) ||
      overlap(v_cache, ncache, M, nM) || overlap(M, nM, z, nz))
    return INFINI_ERR_ALIAS;
  int dev = 0, sms = 148;
  if (prepare_device(&dev) != cudaSuccess) return INFINI_ERR_CUDA;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  Scratch sp;
  int st = get_scratch(sp, bf16_decode_workspace_bytes((int)BH, n, pos, sms), nullptr, stream);
  if (st != INFINI_OK) return st;
  const auto* kcb = static_cast<const __nv_bfloat16*>(k_cache);
  const auto* vcb = static_cast<const __nv_bfloat16*>(v_cache);
  if (bf16_decode_launch(static_cast<const __nv_bfloat16*>(q),
                         static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
                         static_cast<__nv_bfloat16*>(k_cache), static_cast<__nv_bfloat16*>(v_cache),
                         beta, M, z, static_cast<__nv_bfloat16*>(out), static_cast<float*>(sp.ptr),
                         (int)BH, H, n, pos, N, sms, stream) != cudaSuccess)
    return INFINI_ERR_CUDA;
  if (pos + n < N) return INFINI_OK;
  // the completed segment's update, in place: the one-segment state kernel over the
  // cache (token chunks in parallel, the chunks added to M in chunk order)
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  int sCH = 1, sCL = N;
  bf16_step_state_plan((int)BH, N, &sCH, &sCL);
  const size_t state_bytes = up(bf16_workspace_bytes((int)BH, 1, 1));
  Scratch sc;
  st = get_scratch(sc, state_bytes + bf16_step_state_bytes((int)BH, sCH), nullptr, stream);
  if (st != INFINI_OK) return st;
  const Bf16Workspace ws = bf16_workspace_carve(sc.ptr, (int)BH, 1, 1);
  void* step_ws = static_cast<char*>(sc.ptr) + state_bytes;
  cudaError_t e = bf16_prep_first(M, z, ws, (int)BH, 1, stream,
                                  bf16_step_state_counters(step_ws, (int)BH, sCH), 2 * (int)BH);
  if (e == cudaSuccess)
    e = bf16_step_state_launch(kcb, vcb, M, M, z, ws, step_ws, (int)BH, N, sCH, sCL, mode, stream);
  return e == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

// Gradient of the bf16 forward: the state path rebuilds every segment's incoming
// state, then the backward kernels (bf16_bwd.cu) run in order on the caller's stream.
int backward_impl(const void* q, const void* k, const void* v, const float* beta,
                  const float* M_in, const float* z_in, const void* dout, const float* dM_out,
                  const float* dz_out, void* dq, void* dk, void* dv, float* dbeta, float* dM_in,
                  float* dz_in, int B, int H, long long L, int N, int d, int mode,
                  const infini_attn_opts_t* opts, cudaStream_t stream) {
  if (!beta || !dbeta) return INFINI_ERR_NULL;
  if (L > 0 && (!q || !k || !v || !dout || !dq || !dk || !dv)) return INFINI_ERR_NULL;
  if ((M_in == nullptr) != (z_in == nullptr)) return INFINI_ERR_NULL;
  if ((dM_out == nullptr) != (dz_out == nullptr)) return INFINI_ERR_NULL;
  if ((dM_in == nullptr) != (dz_in == nullptr)) return INFINI_ERR_NULL;
  if (B < 1 || H < 1 || N < 1 || L < 0 || d < 1) return INFINI_ERR_SHAPE;
  if (mode != INFINI_LINEAR && mode != INFINI_DELTA) return INFINI_ERR_UNSUPPORTED;
  if (d != 128 || N % 128 != 0 || L % N != 0) return INFINI_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  if (BH > (1LL << 30) || overflows(BH, L) || overflows(BH * L, (long long)d * 4) ||
      L >= (1LL << 31))
    return INFINI_ERR_SHAPE;
  const void* tok[] = {q, k, v, dout, dq, dk, dv};
  for (const void* p : tok)
    if (L > 0 && !aligned16(p)) return INFINI_ERR_ALIGN;
  const void* st_ptrs[] = {M_in, z_in, dM_out, dz_out, dM_in, dz_in};
  for (const void* p : st_ptrs)
    if (p && !aligned16(p)) return INFINI_ERR_ALIGN;
  const size_t nio = (size_t)(BH * L * d) * 2;
  const size_t nM = (size_t)BH * d * d * sizeof(float), nz = (size_t)BH * d * sizeof(float);
  const size_t nb = (size_t)H * sizeof(float);
  const void* ins[] = {q, k, v, dout, M_in, z_in, dM_out, dz_out, beta};
  const size_t in_n[] = {nio, nio, nio, nio, nM, nz, nM, nz, nb};
  void* outs[] = {dq, dk, dv, dM_in, dz_in, dbeta};
  const size_t out_n[] = {nio, nio, nio, nM, nz, nb};
  for (int a = 0; a < 6; ++a) {
    if (L == 0 && a < 3) continue;
    for (int c = 0; c < 9; ++c)
      if (overlap(outs[a], out_n[a], ins[c], in_n[c])) return INFINI_ERR_ALIAS;
    for (int c = a + 1; c < 6; ++c)
      if (overlap(outs[a], out_n[a], outs[c], out_n[c])) return INFINI_ERR_ALIAS;
  }
  int dev = 0;
  if (prepare_device(&dev) != cudaSuccess) return INFINI_ERR_CUDA;
  if (L == 0) {
    // no tokens: the state passes through unchanged, beta has no influence
    if (cudaMemsetAsync(dbeta, 0, nb, stream) != cudaSuccess) return INFINI_ERR_CUDA;
    return pass_state(dM_out, dz_out, dM_in, dz_in, BH, d, stream);
  }
  const int S = (int)(L / N), T = N / 128;
  int CH = 1, CL = N;
  bf16_state_plan((int)BH, S, N, &CH, &CL);
  if (BH * S * CH >= (1LL << 31) || BH * S * T >= (1LL << 31)) return INFINI_ERR_SHAPE;
  Scratch sc;
  const int st = get_scratch(sc, bf16_bwd_workspace_bytes((int)BH, L, S, T, CH), opts, stream);
  if (st != INFINI_OK) return st;
  cudaEvent_t ev[3] = {nullptr, nullptr, nullptr};
  if (opts)
    for (int i = 0; i < 3; ++i) ev[i] = static_cast<cudaEvent_t>(opts->stage_events[i]);
  const cudaError_t e = bf16_backward_launch(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), beta, M_in, z_in,
      static_cast<const __nv_bfloat16*>(dout), dM_out, dz_out, static_cast<__nv_bfloat16*>(dq),
      static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv), dbeta, dM_in, dz_in, B, H,
      L, N, mode, sc.ptr, CH, CL, stream, ev);
  return e == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

int gemm_checks(const void* A, const void* Bm, const void* C, long long M, int N, int K) {
  if (!A || !Bm || !C) return INFINI_ERR_NULL;
  if (M < 1 || N < 1 || K < 1) return INFINI_ERR_SHAPE;
  if (M >= (1LL << 31)) return INFINI_ERR_SHAPE;  // tensor-map row coordinates are 32-bit
  if (M % 128 || N % 128 || K % 128) return INFINI_ERR_UNSUPPORTED;
  if (overflows(M, K) || overflows(M * K, 2) || overflows(M, N) || overflows(M * N, 2) ||
      overflows((long long)K, (long long)N * 2) || M / 128 * (N / 128) >= (1LL << 31))
    return INFINI_ERR_SHAPE;
  if (!aligned16(A) || !aligned16(Bm) || !aligned16(C)) return INFINI_ERR_ALIGN;
  if (overlap(C, (size_t)(M * N) * 2, A, (size_t)(M * K) * 2) ||
      overlap(C, (size_t)(M * N) * 2, Bm, (size_t)K * N * 2))
    return INFINI_ERR_ALIAS;
  return INFINI_OK;
}

// One attention layer: q, k, v = x W_Q, x W_K, x W_V ([B, L, heads * d], the heads'
// columns side by side, read in place as [B, L, heads, d]; the three products in one
// GEMM launch when every width is a multiple of 256), the grouped-head forward,
// y = [A_1 ... A_H] W_O.
int layer_forward_impl(const void* x, const void* Wq, const void* Wk, const void* Wv,
                       const void* Wo, const float* beta, const float* M_in, const float* z_in,
                       void* y, float* M_out, float* z_out, int B, long long L, int D_model,
                       int H, int H_kv, int N, int d, int mode, const infini_attn_opts_t* opts,
                       cudaStream_t stream) {
  if (!x || !Wq || !Wk || !Wv || !Wo || !beta || !y) return INFINI_ERR_NULL;
  if ((M_in == nullptr) != (z_in == nullptr) || (M_out == nullptr) != (z_out == nullptr))
    return INFINI_ERR_NULL;
  if (B < 1 || L < 1 || D_model < 1 || H < 1 || H_kv < 1 || N < 1 || d < 1)
    return INFINI_ERR_SHAPE;
  if (H % H_kv != 0) return INFINI_ERR_SHAPE;
  if (mode != INFINI_LINEAR && mode != INFINI_DELTA) return INFINI_ERR_UNSUPPORTED;
  if (d != 128 || D_model % 128 != 0 || ((long long)B * L) % 128 != 0)
    return INFINI_ERR_UNSUPPORTED;
  const long long rows = (long long)B * L;
  if (overflows(rows, (long long)H * d * 2) || overflows(rows, (long long)D_model * 2) ||
      L >= (1LL << 31) || rows >= (1LL << 31))  // the projections' row coordinates are 32-bit
    return INFINI_ERR_SHAPE;
  const void* ins[] = {x, Wq, Wk, Wv, Wo};
  for (const void* q : ins)
    if (!aligned16(q)) return INFINI_ERR_ALIGN;
  if (!aligned16(y) || (M_in && !aligned16(M_in)) || (M_out && !aligned16(M_out)))
    return INFINI_ERR_ALIGN;
  const size_t ny = (size_t)(rows * D_model) * 2;
  const size_t nw_qo = (size_t)D_model * H * d * 2, nw_kv = (size_t)D_model * H_kv * d * 2;
  if (overlap(y, ny, x, ny) || overlap(y, ny, Wq, nw_qo) || overlap(y, ny, Wk, nw_kv) ||
      overlap(y, ny, Wv, nw_kv) || overlap(y, ny, Wo, nw_qo))
    return INFINI_ERR_ALIAS;
  int dev = 0;
  if (prepare_device(&dev) != cudaSuccess) return INFINI_ERR_CUDA;
  const size_t nq = (size_t)(rows * H * d), nkv = (size_t)(rows * H_kv * d);
  // the projections' outputs, then the forward's own scratch
  const size_t proj_bytes = ((2 * nq + 2 * nkv) * 2 + 255) & ~(size_t)255;
  const int S = (int)((L + N - 1) / N);
  const size_t fwd_bytes = fwd_plan(B * H, B * H_kv, S, N, L).bytes;
  Scratch sc;
  infini_attn_opts_t ws_opts;
  memset(&ws_opts, 0, sizeof(ws_opts));
  if (opts) ws_opts.workspace = opts->workspace, ws_opts.workspace_bytes = opts->workspace_bytes;
  const int st = get_scratch(sc, proj_bytes + fwd_bytes, opts ? &ws_opts : nullptr, stream);
  if (st != INFINI_OK) return st;
  infini_attn_opts_t fwd_opts;
  memset(&fwd_opts, 0, sizeof(fwd_opts));
  fwd_opts.workspace = static_cast<char*>(sc.ptr) + proj_bytes;
  fwd_opts.workspace_bytes = fwd_bytes;
  auto* q = static_cast<__nv_bfloat16*>(sc.ptr);
  __nv_bfloat16* k = q + nq;
  __nv_bfloat16* v = k + nkv;
  __nv_bfloat16* a = v + nkv;  // the heads' outputs, [B, L, H, d]
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  cudaError_t e;
  if ((H * d) % 256 == 0 && (H_kv * d) % 256 == 0) {
    // the three projections of x in one launch (x fetched once per 128-row block)
    const __nv_bfloat16* Ws[3] = {static_cast<const __nv_bfloat16*>(Wq),
                                  static_cast<const __nv_bfloat16*>(Wk),
                                  static_cast<const __nv_bfloat16*>(Wv)};
    __nv_bfloat16* Cs[3] = {q, k, v};
    const int Ns[3] = {H * d, H_kv * d, H_kv * d};
    e = bf16_gemm_grouped_launch(xb, Ws, Cs, Ns, 3, rows, D_model, stream);
  } else {
    e = bf16_gemm_launch(xb, static_cast<const __nv_bfloat16*>(Wq), q, rows, H * d, D_model,
                         stream);
    if (e == cudaSuccess)
      e = bf16_gemm_launch(xb, static_cast<const __nv_bfloat16*>(Wk), k, rows, H_kv * d, D_model,
                           stream);
    if (e == cudaSuccess)
      e = bf16_gemm_launch(xb, static_cast<const __nv_bfloat16*>(Wv), v, rows, H_kv * d, D_model,
                           stream);
  }
  if (e != cudaSuccess) return INFINI_ERR_CUDA;
  record(opts, 0, stream);
  const int fs = forward_impl(q, k, v, beta, M_in, z_in, a, M_out, z_out, B, H, L, N, d, mode,
                              INFINI_DTYPE_BF16, fwd_bytes ? &fwd_opts : nullptr, stream, H_kv,
                              INFINI_LAYOUT_BLHD);
  if (fs != INFINI_OK) return fs;
  record(opts, 1, stream);
  e = bf16_gemm_launch(a, static_cast<const __nv_bfloat16*>(Wo), static_cast<__nv_bfloat16*>(y),
                       rows, D_model, H * d, stream);
  record(opts, 2, stream);
  return e == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

}  // namespace
}  // namespace infini

using namespace infini;

extern "C" {

int infini_attn_forward(const void* q, const void* k, const void* v, const float* beta,
                        const float* M_in, const float* z_in, void* out, float* M_out,
                        float* z_out, int B, int H, long long L, int N, int d, int mode,
                        void* stream) {
  return forward_impl(q, k, v, beta, M_in, z_in, out, M_out, z_out, B, H, L, N, d, mode,
                      INFINI_DTYPE_BF16, nullptr, static_cast<cudaStream_t>(stream));
}

int infini_attn_step(const void* q, const void* k, const void* v, const float* beta,
                     const float* M_in, const float* z_in, void* out, float* M_out,
                     float* z_out, int B, int H, int N, int d, int mode, void* stream) {
  return forward_impl(q, k, v, beta, M_in, z_in, out, M_out, z_out, B, H, N, N < 1 ? 1 : N, d,
                      mode, INFINI_DTYPE_BF16, nullptr, static_cast<cudaStream_t>(stream));
}

int infini_attn_forward_f32(const float* q, const float* k, const float* v, const float* beta,
                            const float* M_in, const float* z_in, float* out, float* M_out,
                            float* z_out, int B, int H, long long L, int N, int d, int mode,
                            void* stream) {
  return forward_impl(q, k, v, beta, M_in, z_in, out, M_out, z_out, B, H, L, N, d, mode,
                      INFINI_DTYPE_F32, nullptr, static_cast<cudaStream_t>(stream));
}

int infini_attn_step_f32(const float* q, const float* k, const float* v, const float* beta,
                         const float* M_in, const float* z_in, float* out, float* M_out,
                         float* z_out, int B, int H, int N, int d, int mode, void* stream) {
  return forward_impl(q, k, v, beta, M_in, z_in, out, M_out, z_out, B, H, N, N < 1 ? 1 : N, d,
                      mode, INFINI_DTYPE_F32, nullptr, static_cast<cudaStream_t>(stream));
}

int infini_attn_forward_gqa(const void* q, const void* k, const void* v, const float* beta,
                            const float* M_in, const float* z_in, void* out, float* M_out,
                            float* z_out, int B, int H, int H_kv, long long L, int N, int d,
                            int mode, int layout, void* stream) {
  if (H_kv < 1) return INFINI_ERR_SHAPE;
  return forward_impl(q, k, v, beta, M_in, z_in, out, M_out, z_out, B, H, L, N, d, mode,
                      INFINI_DTYPE_BF16, nullptr, static_cast<cudaStream_t>(stream), H_kv, layout);
}

int infini_attn_state_sum(const float* dM, const float* dz, int count, const float* M_in,
                          const float* z_in, float* M_out, float* z_out, int B, int H, int d,
                          void* stream) {
  if (!M_out || !z_out || (count > 0 && (!dM || !dz))) return INFINI_ERR_NULL;
  if ((M_in == nullptr) != (z_in == nullptr)) return INFINI_ERR_NULL;
  if (B < 1 || H < 1 || d < 1 || count < 0) return INFINI_ERR_SHAPE;
  const long long BH = (long long)B * H;
  if (BH > (1LL << 30) || overflows(BH * d, (long long)d) || overflows(BH * d * d, (long long)count + 1))
    return INFINI_ERR_SHAPE;
  const long long nM = BH * d * d, nz = BH * d;
  const size_t bM = (size_t)nM * sizeof(float), bz = (size_t)nz * sizeof(float);
  if (overlap(M_out, bM, dM, bM * count) || overlap(M_out, bM, dz, bz * count) ||
      overlap(z_out, bz, dM, bM * count) || overlap(z_out, bz, dz, bz * count) ||
      overlap(M_out, bM, z_out, bz))
    return INFINI_ERR_ALIAS;
  int dev = 0;
  if (prepare_device(&dev) != cudaSuccess) return INFINI_ERR_CUDA;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  state_sum_kernel<<<(unsigned)min((nM + 255) / 256, 4096LL), 256, 0, st>>>(dM, dz, count, M_in,
                                                                           z_in, M_out, z_out,
                                                                           nM, nz);
  return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

int infini_attn_state_update(const void* k, const void* v, const float* M_in, const float* z_in,
                             float* M_out, float* z_out, int B, int H, long long L, int N, int d,
                             int mode, void* stream) {
  return state_update_impl(k, v, M_in, z_in, M_out, z_out, B, H, L, N, d, mode,
                           static_cast<cudaStream_t>(stream));
}

int infini_attn_decode(const void* q, const void* k, const void* v, const float* beta,
                       void* k_cache, void* v_cache, float* M, float* z, void* out, int B, int H,
                       int n, int pos, int N, int d, int mode, void* stream) {
  return decode_impl(q, k, v, beta, k_cache, v_cache, M, z, out, B, H, n, pos, N, d, mode,
                     static_cast<cudaStream_t>(stream));
}

size_t infini_attn_workspace_size(int B, int H, long long L, int N, int d, int mode, int dtype) {
  (void)mode;
  if (B < 1 || H < 1 || N < 1 || L <= 0 || d < 1) return 0;
  const int BH = B * H;
  const int S = (int)((L + N - 1) / N);
  if (dtype == INFINI_DTYPE_F32) return f32_workspace_bytes(BH, S, d);
  return fwd_plan(BH, BH, S, N, L).bytes;
}

int infini_attn_forward_ex(const void* q, const void* k, const void* v, const float* beta,
                           const float* M_in, const float* z_in, void* out, float* M_out,
                           float* z_out, int B, int H, long long L, int N, int d, int mode,
                           int dtype, const infini_attn_opts_t* opts, void* stream) {
  return forward_impl(q, k, v, beta, M_in, z_in, out, M_out, z_out, B, H, L, N, d, mode, dtype,
                      opts, static_cast<cudaStream_t>(stream));
}

int infini_attn_backward(const void* q, const void* k, const void* v, const float* beta,
                         const float* M_in, const float* z_in, const void* dout,
                         const float* dM_out, const float* dz_out, void* dq, void* dk, void* dv,
                         float* dbeta, float* dM_in, float* dz_in, int B, int H, long long L,
                         int N, int d, int mode, void* stream) {
  return backward_impl(q, k, v, beta, M_in, z_in, dout, dM_out, dz_out, dq, dk, dv, dbeta, dM_in,
                       dz_in, B, H, L, N, d, mode, nullptr, static_cast<cudaStream_t>(stream));
}

int infini_attn_backward_ex(const void* q, const void* k, const void* v, const float* beta,
                            const float* M_in, const float* z_in, const void* dout,
                            const float* dM_out, const float* dz_out, void* dq, void* dk,
                            void* dv, float* dbeta, float* dM_in, float* dz_in, int B, int H,
                            long long L, int N, int d, int mode, const infini_attn_opts_t* opts,
                            void* stream) {
  return backward_impl(q, k, v, beta, M_in, z_in, dout, dM_out, dz_out, dq, dk, dv, dbeta, dM_in,
                       dz_in, B, H, L, N, d, mode, opts, static_cast<cudaStream_t>(stream));
}

size_t infini_attn_backward_workspace_size(int B, int H, long long L, int N, int d, int mode) {
  (void)mode;
  if (B < 1 || H < 1 || N < 128 || L <= 0 || d != 128 || N % 128 != 0 || L % N != 0) return 0;
  const long long BH = (long long)B * H;
  if (BH > (1LL << 30) || L >= (1LL << 31)) return 0;
  const int S = (int)(L / N);
  int CH = 1, CL = N;
  bf16_state_plan((int)BH, S, N, &CH, &CL);
  return bf16_bwd_workspace_bytes((int)BH, L, S, N / 128, CH);
}

int infini_attn_gemm_bf16(const void* A, const void* B, void* C, long long M, int N, int K,
                          void* stream) {
  const int st = gemm_checks(A, B, C, M, N, K);
  if (st != INFINI_OK) return st;
  int dev = 0;
  if (prepare_device(&dev) != cudaSuccess) return INFINI_ERR_CUDA;
  const cudaError_t e = bf16_gemm_launch(static_cast<const __nv_bfloat16*>(A),
                                         static_cast<const __nv_bfloat16*>(B),
                                         static_cast<__nv_bfloat16*>(C), M, N, K,
                                         static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

int infini_attn_layer_forward(const void* x, const void* Wq, const void* Wk, const void* Wv,
                              const void* Wo, const float* beta, const float* M_in,
                              const float* z_in, void* y, float* M_out, float* z_out, int B,
                              long long L, int D_model, int H, int H_kv, int N, int d, int mode,
                              void* stream) {
  return layer_forward_impl(x, Wq, Wk, Wv, Wo, beta, M_in, z_in, y, M_out, z_out, B, L, D_model,
                            H, H_kv, N, d, mode, nullptr, static_cast<cudaStream_t>(stream));
}

int infini_attn_layer_forward_ex(const void* x, const void* Wq, const void* Wk, const void* Wv,
                                 const void* Wo, const float* beta, const float* M_in,
                                 const float* z_in, void* y, float* M_out, float* z_out, int B,
                                 long long L, int D_model, int H, int H_kv, int N, int d, int mode,
                                 const infini_attn_opts_t* opts, void* stream) {
  return layer_forward_impl(x, Wq, Wk, Wv, Wo, beta, M_in, z_in, y, M_out, z_out, B, L, D_model,
                            H, H_kv, N, d, mode, opts, static_cast<cudaStream_t>(stream));
}

size_t infini_attn_layer_workspace_size(int B, long long L, int D_model, int H, int H_kv, int N,
                                        int d, int mode) {
  (void)mode;
  (void)D_model;
  if (B < 1 || L < 1 || H < 1 || H_kv < 1 || N < 1 || d != 128 || H % H_kv != 0) return 0;
  const long long rows = (long long)B * L;
  if (rows % 128 != 0 || L >= (1LL << 31) || rows >= (1LL << 31) ||
      overflows(rows, (long long)H * d * 2))
    return 0;
  const size_t nq = (size_t)(rows * H * d), nkv = (size_t)(rows * H_kv * d);
  const size_t proj_bytes = ((2 * nq + 2 * nkv) * 2 + 255) & ~(size_t)255;
  const int S = (int)((L + N - 1) / N);
  return proj_bytes + fwd_plan(B * H, B * H_kv, S, N, L).bytes;
}

int infini_attn_device_status(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return INFINI_ERR_CUDA;
  int flag = 0;
  if (cudaMemcpyFromSymbol(&flag, g_device_error, sizeof(int)) != cudaSuccess)
    return INFINI_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess)
    return INFINI_ERR_CUDA;
  return flag == kDevErrTimeout ? INFINI_ERR_TIMEOUT : INFINI_OK;
}

int infini_attn_selftest_timeout(long long timeout_ns, void* stream) {
  if (timeout_ns < 0 || timeout_ns > 10000000000LL) return INFINI_ERR_SHAPE;
  timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      (unsigned long long)timeout_ns);
  return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

const char* infini_attn_strerror(int status) {
  switch (status) {
    case INFINI_OK: return "ok";
    case INFINI_ERR_NULL: return "a required pointer is NULL (or M/z NULL-ness differs)";
    case INFINI_ERR_SHAPE: return "invalid or overflowing sizes";
    case INFINI_ERR_UNSUPPORTED: return "unsupported head width, mode or dtype";
    case INFINI_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case INFINI_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case INFINI_ERR_NOMEM: return "scratch memory could not be obtained";
    case INFINI_ERR_TIMEOUT: return "a bounded device wait ran out";
    case INFINI_ERR_ALIAS: return "out overlaps an input or the state";
    case INFINI_ERR_SCRATCH_LIMIT: return "sizes need more scratch than the fixed static array holds";
    default: return "unknown status";
  }
}

int infini_attn_version(void) { return 100; }

}  // extern "C"
