// step_static.cu — infini_attn_step_static: the bf16 streaming step without any
// device-memory allocation.
//
// Why it exists: some callers must not allocate device memory while they run.
// A serving loop that reserved its whole memory budget at start-up, a framework
// whose own allocator owns every byte of device memory (a raw cudaMalloc or a
// stream-ordered allocation would sit outside its accounting and can fail or
// fragment the heap), or a runtime with a hard, fixed memory plan cannot let the
// library take scratch space behind its back. This entry point runs the same
// kernels as infini_attn_step, but their scratch lives in one fixed array,
// reserved when the library is loaded, so the call itself allocates nothing.
//
// Rules of use:
//   * The array (kStepScratchBytes = 8 MiB) exists once per device for the life
//     of the process, on every GPU that loads the library.
//   * The first call on a device looks up the array's device address (and sets
//     the kernels' shared-memory limits) for that device; make that first call
//     before any stream capture begins.
//   * Every call on a device uses the same array and leaves its contents behind.
//     The kernels fully overwrite what they read, so nothing needs clearing
//     between calls, but calls whose GPU work overlaps in time (different
//     streams, no ordering between them) race on the array: order them on one
//     stream or synchronise them.
//   * Sizes whose scratch does not fit are rejected with
//     INFINI_ERR_SCRATCH_LIMIT before anything is launched.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <mutex>

#include "infini_attn.h"
#include "bf16_path.h"

namespace infini {

cudaError_t bf16_state_set_attributes();
cudaError_t bf16_attn_set_attributes();

namespace {

constexpr size_t kStepScratchBytes = 8u << 20;  // 8 MiB per device
static __device__ __align__(256) unsigned char g_step_scratch[kStepScratchBytes];

constexpr int kMaxDev = 64;
void* g_scratch_ptr[kMaxDev] = {};
std::mutex g_scratch_mu;

// Device address of the array on the current device (looked up once per device,
// with that device current). Returns nullptr on failure.
void* scratch_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_step_scratch) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    if (bf16_state_set_attributes() != cudaSuccess || bf16_attn_set_attributes() != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace infini

using namespace infini;

extern "C" int infini_attn_step_static(const void* q, const void* k, const void* v,
                                       const float* beta, const float* M_in, const float* z_in,
                                       void* out, float* M_out, float* z_out, int B, int H,
                                       int N, int d, int mode, void* stream) {
  if (!beta) return INFINI_ERR_NULL;
  if (N > 0 && (!q || !k || !v || !out)) return INFINI_ERR_NULL;
  if ((M_in == nullptr) != (z_in == nullptr)) return INFINI_ERR_NULL;
  if ((M_out == nullptr) != (z_out == nullptr)) return INFINI_ERR_NULL;
  if (B < 1 || H < 1 || N < 1) return INFINI_ERR_SHAPE;
  if ((long long)B * H > (1LL << 30)) return INFINI_ERR_SHAPE;
  if (mode != INFINI_LINEAR && mode != INFINI_DELTA) return INFINI_ERR_UNSUPPORTED;
  if (d != 128) return INFINI_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return INFINI_ERR_ALIGN;
  if ((M_in && !aligned16(M_in)) || (M_out && !aligned16(M_out))) return INFINI_ERR_ALIGN;
  // out may overlap none of the inputs and none of the state buffers (the same rule
  // as infini_attn_step)
  const size_t nio = (size_t)B * H * N * d * 2;
  const size_t nM = (size_t)B * H * d * d * sizeof(float), nz = (size_t)B * H * d * sizeof(float);
  const uintptr_t o = reinterpret_cast<uintptr_t>(out);
  const struct {
    const void* p;
    size_t n;
  } others[] = {{q, nio}, {k, nio}, {v, nio}, {M_in, nM}, {z_in, nz}, {M_out, nM}, {z_out, nz}};
  for (const auto& x : others) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(x.p);
    if (x.p && o < a + x.n && a < o + nio) return INFINI_ERR_ALIAS;
  }

  // Token chunking of the state GEMM: as in the allocating call, but halved
  // until the scratch fits the fixed array.
  const int BH = B * H, S = 1;
  int CH = 1, CL = N;
  bf16_state_plan(BH, S, N, &CH, &CL);
  while (CH > 1 && bf16_workspace_bytes(BH, S, CH) > kStepScratchBytes) {
    CH /= 2;
    CL = (N + CH - 1) / CH;
  }
  if (bf16_workspace_bytes(BH, S, CH) > kStepScratchBytes) return INFINI_ERR_SCRATCH_LIMIT;

  void* scratch = scratch_for_current_device();
  if (!scratch) return INFINI_ERR_CUDA;
  const Bf16Workspace ws = bf16_workspace_carve(scratch, BH, S, CH);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto* kb = static_cast<const __nv_bfloat16*>(k);
  const auto* vb = static_cast<const __nv_bfloat16*>(v);
  if (bf16_state_launch(kb, vb, M_in, z_in, M_out, z_out, ws, BH, N, N, S, CH, CL, mode, 0, st) !=
      cudaSuccess)
    return INFINI_ERR_CUDA;
  if (bf16_attn_launch(static_cast<const __nv_bfloat16*>(q), kb, vb, beta,
                       static_cast<__nv_bfloat16*>(out), ws, BH, H, N, N, S, st) != cudaSuccess)
    return INFINI_ERR_CUDA;
  return INFINI_OK;
}
