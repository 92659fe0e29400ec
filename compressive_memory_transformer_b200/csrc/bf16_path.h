// bf16_path.h — internal interface of the bf16 forward (d = 128): the state
// kernels (bf16_state.cu) and the fused attention kernel (bf16_attn.cu).
#pragma once
#include <cstddef>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace infini {

// Scratch of one bf16 forward call, carved from one allocation.
//   zpart [BH][S][CH][128] f32   partial sums of sigma(K) per token chunk
//   zprev [BH][S][128]     f32   z_{s-1} for every segment
//   dpart [BH][S][CH][2][128][128] f32   per-chunk [dM | G] of the state GEMM
//   Mhl   [BH][S][2][128][128] bf16      M_{s-1} as hi and lo bf16 parts
struct Bf16Workspace {
  float* zpart;
  float* zprev;
  float* dpart;
  __nv_bfloat16* Mhl;
};

// Where q/k/v/out sit: element (b, h, l, f) of q and out at b*q_sb + h*q_sh + l*q_sl + f,
// of k and v at b*kv_sb + h*kv_sh + l*kv_sl + f (strides in elements). H query heads
// share H_kv key/value heads (query head h reads key/value head h / (H / H_kv)); the
// memory state is per key/value head. bhld() is the contiguous [B, H, L, d] case.
struct Bf16Layout {
  int B, H, H_kv;
  long long q_sb, q_sh, q_sl, kv_sb, kv_sh, kv_sl;
  static Bf16Layout bhld(int B, int H, long long L) {
    const long long d = 128;
    return Bf16Layout{B, H, H, (long long)H * L * d, L * d, d, (long long)H * L * d, L * d, d};
  }
  static Bf16Layout blhd(int B, int H, int H_kv, long long L) {
    const long long d = 128;
    return Bf16Layout{B, H, H_kv, L * H * d, d, (long long)H * d, L * H_kv * d, d,
                      (long long)H_kv * d};
  }
};

void bf16_state_plan(int BH, int S, int N, int* CH, int* CL);
size_t bf16_workspace_bytes(int BH, int S, int CH);
Bf16Workspace bf16_workspace_carve(void* base, int BH, int S, int CH);

// The state path. Segments s < first (0 or 1) of the workspace's M_{s-1} hi/lo
// and z_{s-1} are taken as already written (by bf16_prep_first) and not rewritten.
// BH here counts key/value heads (B * H_kv); k and v are read through the layout.
cudaError_t bf16_state_launch(const __nv_bfloat16* k, const __nv_bfloat16* v, const float* M_in,
                              const float* z_in, float* M_out, float* z_out,
                              const Bf16Workspace& ws, int BH, long long L, int N, int S, int CH,
                              int CL, int mode, int first, cudaStream_t stream,
                              const Bf16Layout* lay = nullptr);

// Writes the workspace's first-segment M_{-1} hi/lo and z_{-1} from M_in / z_in, and
// zeroes ctr[0 .. nctr) (counters of kernels launched after it).
cudaError_t bf16_prep_first(const float* M_in, const float* z_in, const Bf16Workspace& ws,
                            int BH, int S, cudaStream_t stream, unsigned* ctr = nullptr,
                            int nctr = 0);

// The memory update of a call holding one segment (bf16_step_state.cu): CTAs per (head,
// token chunk, column block) compute sigma(K)^T (V - sigma(K) M_in / den) in parallel
// and the last CTA of each (head, column block) adds the chunks to M_in in chunk order.
// Reads the workspace's M_{-1} hi/lo and z_{-1} (bf16_prep_first) and k, v; writes
// M_out, z_out. step_ws holds bf16_step_state_bytes(BH, CH) bytes whose counters
// (bf16_step_state_counters, 2 * BH of them) are zero at the launch. BH counts key/value
// heads.
void bf16_step_state_plan(int BH, int N, int* CH, int* CL);
size_t bf16_step_state_bytes(int BH, int CH);
unsigned* bf16_step_state_counters(void* step_ws, int BH, int CH);
cudaError_t bf16_step_state_launch(const __nv_bfloat16* k, const __nv_bfloat16* v,
                                   const float* M_in, float* M_out, float* z_out,
                                   const Bf16Workspace& ws, void* step_ws, int BH, int N, int CH,
                                   int CL, int mode, cudaStream_t stream,
                                   const Bf16Layout* lay = nullptr);

// Split mode of the attention kernel, for calls whose query-tile pairs are fewer than
// the SMs (one segment of a few heads, short sequences): each query tile's key range
// is cut into pieces of at most C key tiles, the pieces are taken from a device
// counter heaviest first, and the last piece of a tile to finish merges the pieces'
// partial results (log-sum-exp weights, fixed piece order) into the output.
struct Bf16AttnSplit {
  int C = 0;             // 0: no split (tile pairs dealt out round-robin)
  int Pmax = 0;          // most pieces of one tile
  long long units = 0;   // pieces in the call
};
// BH counts query heads (B * H).
Bf16AttnSplit bf16_attn_split_plan(int BH, int S, int N, long long L, int sms);
// Scratch of a split call (counters and partial records; 0 without a split).
size_t bf16_attn_split_bytes(const Bf16AttnSplit& sp, int BH, int S, int N, long long L);

// The fused local-attention + retrieval + gate kernel. Reads q, k, v, beta and
// the workspace's zprev / Mhl; writes out.
// BH counts query heads (B * H); the workspace holds the key/value heads' states.
// split / split_ws: a split plan and bf16_attn_split_bytes(...) bytes of scratch
// (zeroed counters are set up on `stream` before the kernel); NULL: tile pairs.
cudaError_t bf16_attn_launch(const __nv_bfloat16* q, const __nv_bfloat16* k,
                             const __nv_bfloat16* v, const float* beta, __nv_bfloat16* out,
                             const Bf16Workspace& ws, int BH, int H, long long L, int N, int S,
                             cudaStream_t stream, const Bf16Layout* lay = nullptr,
                             const Bf16AttnSplit* split = nullptr, void* split_ws = nullptr);

// Gradient of the bf16 forward (bf16_bwd.cu): [B, H, L, 128] contiguous, N a multiple
// of 128, L a multiple of N. `scratch` holds bf16_bwd_workspace_bytes(...) bytes; CH /
// CL are the state path's token chunking (bf16_state_plan).
size_t bf16_bwd_workspace_bytes(int BH, long long L, int S, int T, int CH);
cudaError_t bf16_backward_launch(const __nv_bfloat16* q, const __nv_bfloat16* k,
                                 const __nv_bfloat16* v, const float* beta, const float* M_in,
                                 const float* z_in, const __nv_bfloat16* dout,
                                 const float* dM_out, const float* dz_out, __nv_bfloat16* dq,
                                 __nv_bfloat16* dk, __nv_bfloat16* dv, float* dbeta, float* dM_in,
                                 float* dz_in, int B, int H, long long L, int N, int mode,
                                 void* scratch, int CH, int CL, cudaStream_t stream,
                                 cudaEvent_t const* events = nullptr);

// C [M][N] = A [M][K] B [K][N] (bf16, row-major, fp32 accumulation; bf16_gemm.cu);
// M, N, K multiples of 128.
cudaError_t bf16_gemm_launch(const __nv_bfloat16* A, const __nv_bfloat16* B, __nv_bfloat16* C,
                             long long M, int N, int K, cudaStream_t stream);
// C_g = A B_g (g < ngroups <= 3) in one launch: B_g [K][N_g], C_g [M][N_g] row-major, every
// N_g a multiple of 256; each 128-row block of A is fetched once for all the groups.
cudaError_t bf16_gemm_grouped_launch(const __nv_bfloat16* A, const __nv_bfloat16* const* B,
                                     __nv_bfloat16* const* C, const int* N, int ngroups,
                                     long long M, int K, cudaStream_t stream);

// Token-level decode (bf16_decode.cu): partial attention over the KV cache (rows
// below pos) and the new rows (k, v, also written into the caches), split like flash
// decoding, then merge + retrieval from the fp32 state + gate. `part` holds
// bf16_decode_workspace_bytes(...) bytes.
size_t bf16_decode_workspace_bytes(int BH, int n, int pos, int sms);
cudaError_t bf16_decode_launch(const __nv_bfloat16* q, const __nv_bfloat16* k,
                               const __nv_bfloat16* v, __nv_bfloat16* k_cache,
                               __nv_bfloat16* v_cache, const float* beta, const float* M,
                               const float* z, __nv_bfloat16* out, float* part, int BH, int H,
                               int n, int pos, int N, int sms, cudaStream_t stream);


}  // namespace infini
