// bf16_attn.cu — fused local attention + memory retrieval + gate (bf16, d = 128).
//
// For every 128-row query tile of every segment of every (batch, head):
//   A_dot = softmax(Q K^T / sqrt(d) + causal mask) V     over the segment's keys
//   A_mem = sigma(Q) M_{s-1} / (sigma(Q) z_{s-1})         (0 where the denominator is 0)
//   out   = g A_mem + (1 - g) A_dot,  g = sigmoid(beta_h)
// ("Leave No Context Behind", arXiv 2404.07143, as quoted on
// llm-papers-study.pages.dev: sections 3.1, 3.3, 3.5). A_dot and A_mem stay in
// tensor memory; only `out` is written to HBM.
//
// Persistent kernel: one CTA per SM walks a list of work units. A unit is a pair
// of query tiles of one segment, i and T-1-i (T tiles per segment), so every unit
// holds T+1 key tiles of work; units are dealt out round-robin in segment order,
// so the ~150 units in flight touch ~20 segments and their K/V stay in L2.
// Every pipeline runs on across tiles: while the softmax warps finish one tile,
// the producer already loads the next Q (prefetched into L2 a tile earlier) and K
// tiles and the next tile's first Q K^T products are issued.
//
// Warp roles (352 threads):
//   warp 0     TMA producer: Q per tile (reloaded once the last Q K^T of the tile
//              and sigma(Q) are done) together with the tile's descriptor (a shared
//              memory slot, so no other role walks the work list); a K ring (2
//              stages); a V ring (2 stages) whose items per tile are M_hi (the
//              state rounded to bf16), then V_0, V_1, ...
//   warp 1     tensor-memory allocation; issues the retrieval and P V products.
//   warp 10    issues the Q K^T products (another scheduler than warp 1, so each
//              issuing warp carries half of the per-key-tile instruction stream).
//   warps 2-9  softmax / epilogue, two warpgroups: query row r (tensor-memory lane r)
//              is shared by one thread of each; warpgroup h owns key columns
//              [64h, 64h + 64) of S and value columns [64h, 64h + 64) of O, R and out.
//              The two threads of a row exchange their partial row max every key
//              tile (and row sum / denominator at the end) through shared memory,
//              synchronised by an mbarrier per warp pair. Softmax barriers count
//              one arrival per warp.
// Tensor memory (512 columns): S0 | S1 (scores, alternating over the global key-tile
// sequence) | O (A_dot accumulator) | R (sigma(Q) M accumulator). P (bf16) is
// written over the first 64 columns of its S buffer and read from there by the PV
// MMA; sigma(Q) (bf16) is staged in O, each half in its own columns, for the
// retrieval MMA before the tile's first PV overwrites O.
// Tensor-core operations from one issuing thread execute in issue order: warp 1's
// retrieval precedes the tile's first P V (which overwrites the staged sigma(Q)).
// Across the two issuing warps the order is explicit: the Q K^T of key step n
// overwrites the S buffer that held P of step n - 2, so it waits for that step's
// P V through the buffer's S-free barrier.
// Every mbarrier is waited on in completion order and can never complete twice
// before its waiter has seen the first completion (a parity wait would then
// miss it): sigma(Q) and P have separate barriers; P has one per S buffer (P of
// step n + 2 needs the S of step n + 2, whose Q K^T waited for the P V of step n);
// the next tile's sigma(Q) is written only after the epilogue saw R and the last
// P V done. The softmax warps wait for a P V (through its S buffer's S-free
// barrier) only before touching O: for a rescale, and in the epilogue.
// z_{s-1} (512 B) rides on the Q barrier.
// Online softmax keeps a per-row reference max and rescales O only when the
// running max grows by more than 2^8 (in exp2 units). One exponential in four is
// evaluated on the FMA pipe (ex2_poly2) to offload the MUFU unit. The retrieval
// uses M rounded to one bf16 term: A_mem is a weighted average over the 128 rows
// of M, so the independent per-element roundings (relative 2^-9) average out to
// ~5e-5 of the output, far inside the bf16 output tolerance.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda.h>
#include <cstdint>

#include "bf16_path.h"
#include "sm100.cuh"
#include "tma_map.h"

namespace infini {
namespace {

constexpr int D = 128;
constexpr int BM = 128;   // query rows per tile
constexpr int BN = 128;   // keys per tile
constexpr int kTile = 32768;     // one 128 x 128 bf16 tile
constexpr int kSub = 16384;      // one 128 x 64 box (128-byte rows)
constexpr int kVStages = 2;
constexpr int OFF_Q = 0;
constexpr int OFF_K = kTile;         // 2 stages
constexpr int OFF_V = 3 * kTile;     // kVStages stages
constexpr int OFF_OUT = 5 * kTile;   // output tile staged for the TMA store (half h at h * kSub)
constexpr int OFF_X = 6 * kTile;     // exchange: max [2][2][128], den [2][128], l [2][128]
constexpr int OFF_Z = OFF_X + 4096;   // z_{s-1} of the current tile (128 floats), loaded with Q
constexpr int OFF_BAR = OFF_Z + 512;
constexpr int OFF_SLOT = OFF_BAR + 256;  // two tile descriptors
constexpr int OFF_FLAG = OFF_SLOT + 256;  // split mode: "this piece merges" broadcast
constexpr int kAttnSmem = OFF_FLAG + 16 + 1024;  // + alignment slack
constexpr int kThreads = 352;
constexpr int kSoftmaxThreads = 256;
constexpr int kSoftmaxWarps = 8;
// Split mode: the record a piece leaves for the tile's merge. O (128 rows x 128
// value columns, fp32, unnormalised, against the piece's reference row max) as
// [32 column quads][128 rows] float4, then the reference max and the row sum.
constexpr int kRecO = 128 * 128;
constexpr int kRecFloats = kRecO + 2 * 128;

enum {
  B_QFULL = 0, B_QEMPTY = 1, B_KFULL = 2, B_SFREE = 4 /* 2 */, B_VFULL = 6 /* 3 */, B_VEMPTY = 9 /* 3 */,
  B_SFULL = 12, B_PFULL = 14 /* 2 */, B_DRAIN = 16, B_PAIR = 17 /* 4 */, B_RDONE = 21,
  B_SQFULL = 22, B_OFULL = 23 /* 2 */, B_OFREE = 25 /* 2 */, B_SPLW = 27, B_SPLF = 28,
  B_COUNT = 29
};

struct Params {
  long long L;
  int N, S, H, T, U, BH;
  unsigned units;  // tile pairs: BH * S * U; split mode: pieces (below 2^31)
  FastDiv divU, divS, divH, divG;  // G = H / Hkv query heads per key/value head
  int Hkv;
  long long o_sb, o_sh, o_sl;  // out strides (elements): batch row, head, row
  int out32;    // out is 32-byte aligned: rows are stored as whole 32-byte sectors
  int tma_out;  // out has a TMA map: whole tiles leave through shared memory
  // Split mode (calls with fewer tile pairs than SMs): a unit is a piece of one query
  // tile's key range; units are taken from a device counter, heaviest first.
  int split;
  int C;        // most key tiles per piece
  int Pmax;     // record slots per tile
  unsigned BHS; // BH * S
  FastDiv divBHS;
  unsigned* unit_ctr;  // next unit (zeroed before the launch)
  unsigned* tile_ctr;  // [BHS * T] pieces of each tile finished (zeroed before the launch)
  float* rec;          // [BHS * T * Pmax] records of kRecFloats
};

// One query tile (or, in split mode, one piece of its key range) of the work list
// (valid = 0: the end of the CTA's list).
struct Tile {
  long long seg0;
  int bh, s, i, nkv, q_row, rows_valid, h, valid;
  int b, hk, bhk;  // batch row, key/value head, and its index b * Hkv + hk
  int j0;          // first key tile of the piece (0 outside split mode)
  int np, pc;      // pieces of this tile (1 outside split mode) and this piece's index
  unsigned tid;    // split mode: the tile's index (bh * S + s) * T + i
};

// Fills t for query tile i of segment seg = bh * S + s; false when the tile lies past
// the end of a short final segment.
__device__ __forceinline__ bool fill_tile(const Params& p, unsigned seg, int i, Tile& t) {
  const unsigned bh = p.divS.div(seg);
  t.s = (int)(seg - bh * (unsigned)p.S);
  t.bh = (int)bh;
  t.seg0 = (long long)t.s * p.N;
  const int n_s = (int)min((long long)p.N, p.L - t.seg0);
  const int T_s = (n_s + BM - 1) / BM;
  if (i >= T_s) return false;
  t.i = i;
  t.nkv = i + 1;
  t.j0 = 0;
  t.np = 1;
  t.pc = 0;
  t.tid = seg * (unsigned)p.T + (unsigned)i;
  t.b = (int)p.divH.div((uint32_t)t.bh);
  t.h = t.bh - t.b * p.H;
  t.hk = (int)p.divG.div((uint32_t)t.h);
  t.bhk = t.b * p.Hkv + t.hk;
  t.valid = 1;
  t.q_row = (int)(t.seg0 + (long long)i * BM);
  t.rows_valid = min(BM, n_s - i * BM);
  return true;
}

// Split mode, unit u -> piece. Units are ordered heaviest first: query tiles from the
// last (T - 1, the longest key range) down to 0; tile i's i + 1 key tiles form
// np = ceil((i + 1) / C) pieces of near-equal length; within a tile level, piece
// index, then segment.
__device__ __forceinline__ bool decode_piece(const Params& p, unsigned u, Tile& t) {
  for (int i = p.T - 1; i >= 0; --i) {
    const int np = (i + p.C) / p.C;
    const unsigned cnt = (unsigned)np * p.BHS;
    if (u < cnt) {
      const int pc = (int)p.divBHS.div(u);
      const unsigned seg = u - (unsigned)pc * p.BHS;
      if (!fill_tile(p, seg, i, t)) return false;
      const int j0 = pc * (i + 1) / np, j1 = (pc + 1) * (i + 1) / np;
      t.j0 = j0;
      t.nkv = j1 - j0;
      t.np = np;
      t.pc = pc;
      return true;
    }
    u -= cnt;
  }
  return false;
}

// Walks the CTA's tiles. Tile pairs: units blockIdx.x, blockIdx.x + gridDim.x, ...;
// unit u of a segment holds tiles T-1-u and u (one tile when they coincide); tiles
// past the end of a short final segment are skipped. Split mode: each unit is taken
// from the device counter when the producer is ready to load it (after it has issued
// every copy of the previous unit), never earlier: a CTA that starts late, when the
// SMs of a kernel running beside it free up, still finds the units that no CTA has
// begun.
template <bool kSplit>
struct TileIter {
  unsigned unit;
  int k;  // 0: tile T-1-u, 1: tile u
  __device__ void init(const Params& p) {
    unit = blockIdx.x;
    k = 0;
  }
  __device__ bool next(const Params& p, Tile& t) {
    if (kSplit) {
      for (;;) {
        const unsigned u = atomicAdd(p.unit_ctr, 1u);
        if (u >= p.units) return false;
        if (decode_piece(p, u, t)) return true;
      }
    }
    while (unit < p.units) {
      const unsigned seg = p.divU.div(unit);
      const int u = (int)(unit - seg * (unsigned)p.U);
      const int kk = k;
      if (++k == 2) {
        k = 0;
        unit += gridDim.x;
      }
      const int i = kk == 0 ? p.T - 1 - u : u;
      if (kk == 1 && u >= p.T - 1 - u) continue;  // the pair collapsed to one tile
      if (fill_tile(p, seg, i, t)) return true;
    }
    return false;
  }
  // The tile the next call returns, if known without taking a unit (for prefetching;
  // split mode does not know it).
  __device__ bool peek(const Params& p, Tile& t) const {
    if (kSplit) return false;
    TileIter a = *this;
    return a.next(p, t);
  }
};

// Bounded wait used only while draining after an error: ignores the error flag.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) break;  // 200 ms
  }
}

// K-major operand (rows = M or N index, 64 bf16 of K per 128-byte row, two boxes
// of 64 columns 16 KB apart): k-step kk covers K elements [16 kk, 16 kk + 16).
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int kk) {
  return sdesc(base + (uint32_t)(kk >> 2) * kSub + (uint32_t)(kk & 3) * 32, 16, 1024);
}
// MN-major operand (rows = K index, 64 bf16 of N per 128-byte row, two boxes of
// 64 columns 16 KB apart): k-step kk covers K rows [16 kk, 16 kk + 16).
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t base, int kk) {
  return sdesc(base + (uint32_t)kk * 2048, kSub, 1024);
}
// The same two layouts as offsets added to the descriptor of k-step 0.
__device__ __forceinline__ constexpr uint32_t kdesc_off(int kk) {
  return (uint32_t)((kk >> 2) * (kSub >> 4) + (kk & 3) * 2);
}
__device__ __forceinline__ constexpr uint32_t mndesc_off(int kk) { return (uint32_t)kk * 128u; }

// kSplit: split mode (a separate instantiation, so that the tile-pair kernel carries
// none of its code).
template <bool kSplit>
__global__ void __launch_bounds__(kThreads, 1)
attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_m,
            const __grid_constant__ CUtensorMap tm_o,
            const float* __restrict__ beta, const float* __restrict__ zprev,
            __nv_bfloat16* __restrict__ out, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + OFF_Q;
  uint8_t* sK = smem + OFF_K;
  uint8_t* sV = smem + OFF_V;
  uint8_t* sOut = smem + OFF_OUT;
  float* sX = reinterpret_cast<float*>(smem + OFF_X);
  float* sZ = reinterpret_cast<float*>(smem + OFF_Z);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + B_COUNT);
  // Tile descriptors: the producer writes tile c's into slots[c & 1] before it arms
  // Q's full barrier for that tile (release), and after the last tile it writes an
  // end marker and arrives on the barrier without a copy. The other roles read a
  // slot only after a wait that orders them behind that arrival.
  Tile* slots = reinterpret_cast<Tile*>(smem + OFF_SLOT);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int b = 0; b < B_COUNT; ++b) {
      uint32_t cnt = 1;
      // arrivals are counted per warp (mbar_arrive_warp)
      if (b == B_PFULL || b == B_PFULL + 1 || b == B_SQFULL || b == B_SPLW) cnt = kSoftmaxWarps;
      // Q is free once the tile's last Q K^T is done and every softmax warp has
      // read its rows of Q for sigma(Q)
      if (b == B_QEMPTY) cnt = 1 + kSoftmaxWarps;
      // B_RDONE: one commit per tile (retrieval MMAs)
      if (b >= B_PAIR && b < B_PAIR + 4) cnt = 2;
      if (b == B_DRAIN) cnt = 2;  // one commit from each MMA-issuing warp
      if (b == B_OFULL || b == B_OFULL + 1) cnt = 4;  // the four warps of a half
      mbar_init(&bars[b], cnt);
    }
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_m);
    if (p.tma_out) tma_prefetch_desc(&tm_o);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + 256, tR = tmem + 384;

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0) {
      int q_iss = 0, k_iss[2] = {0, 0}, v_iss[kVStages] = {0, 0};
      uint32_t kst = 0, kph = 0, vst = 0, vph = 0;  // next K / V ring stage and phase
      bool k_wrapped = false, v_wrapped = false;     // every stage used at least once
      bool ok = true;
      auto issue_k = [&](const Tile& t, int j) -> bool {
        // the Q K^T that read this stage signalled the same stage's scores barrier
        if (k_wrapped && !mbar_wait(&bars[B_SFULL + kst], kph ^ 1u)) return false;
        mbar_arrive_expect_tx(&bars[B_KFULL + kst], kTile);
        const int row = (int)(t.seg0 + (long long)(t.j0 + j) * BN);
        uint8_t* dst = sK + kst * kTile;
        tma_load_4d(dst, &tm_k, &bars[B_KFULL + kst], 0, row, t.hk, t.b);
        tma_load_4d(dst + kSub, &tm_k, &bars[B_KFULL + kst], 64, row, t.hk, t.b);
        ++k_iss[kst];
        kph ^= kst;
        k_wrapped |= (kst == 1u);
        kst ^= 1u;
        return true;
      };
      auto issue_v = [&](const Tile& t, int item) -> bool {  // item 0: M_hi; 1+j: V_j
        if (v_wrapped && !mbar_wait(&bars[B_VEMPTY + vst], vph ^ 1u)) return false;
        mbar_arrive_expect_tx(&bars[B_VFULL + vst], kTile);
        uint8_t* dst = sV + vst * kTile;
        if (item == 0) {
          const int zc = (t.bhk * p.S + t.s) * 2;
          tma_load_3d(dst, &tm_m, &bars[B_VFULL + vst], 0, 0, zc);
          tma_load_3d(dst + kSub, &tm_m, &bars[B_VFULL + vst], 64, 0, zc);
        } else {
          const int row = (int)(t.seg0 + (long long)(t.j0 + item - 1) * BN);
          tma_load_4d(dst, &tm_v, &bars[B_VFULL + vst], 0, row, t.hk, t.b);
          tma_load_4d(dst + kSub, &tm_v, &bars[B_VFULL + vst], 64, row, t.hk, t.b);
        }
        ++v_iss[vst];
        if (++vst == (uint32_t)kVStages) {
          vst = 0;
          vph ^= 1u;
          v_wrapped = true;
        }
        return true;
      };
      TileIter<kSplit> it;
      it.init(p);
      Tile t;
      int tc = 0;
      while (ok && it.next(p, t)) {
        if (tc > 0 && !mbar_wait(&bars[B_QEMPTY], (uint32_t)((tc - 1) & 1))) {
          ok = false;
          break;
        }
        slots[tc & 1] = t;
        mbar_arrive_expect_tx(&bars[B_QFULL], kTile + D * 4);
        tma_load_4d(sQ, &tm_q, &bars[B_QFULL], 0, t.q_row, t.h, t.b);
        tma_load_4d(sQ + kSub, &tm_q, &bars[B_QFULL], 64, t.q_row, t.h, t.b);
        bulk_load(sZ, zprev + ((size_t)t.bhk * p.S + t.s) * D, D * 4, &bars[B_QFULL]);
        ++q_iss;
        {  // the next tile's Q has a whole tile of work to reach L2
          Tile tn;
          if (it.peek(p, tn)) {
            tma_prefetch_l2_4d(&tm_q, 0, tn.q_row, tn.h, tn.b);
            tma_prefetch_l2_4d(&tm_q, 64, tn.q_row, tn.h, tn.b);
          }
        }
        ok = issue_k(t, 0) && (t.nkv < 2 || issue_k(t, 1)) && issue_v(t, 0);
        for (int j = 0; ok && j < t.nkv; ++j) {
          // K of step j + 2 (its stage frees when Q K^T_j is done) goes before V_j,
          // whose stage frees one P V later
          if (j + 2 < t.nkv) ok = issue_k(t, j + 2);
          if (ok) ok = issue_v(t, j + 1);
        }
        ++tc;
      }
      // end of the list: a descriptor with valid = 0 and a plain arrival
      if (ok && (tc == 0 || mbar_wait(&bars[B_QEMPTY], (uint32_t)((tc - 1) & 1)))) {
        Tile e;
        e.valid = 0;
        slots[tc & 1] = e;
        mbar_arrive(&bars[B_QFULL]);
      }
      if (!ok) {  // let the copies already issued land before the CTA exits
        if (q_iss > 0) drain_wait(&bars[B_QFULL], (uint32_t)((q_iss - 1) & 1));
        for (int st = 0; st < 2; ++st)
          if (k_iss[st] > 0) drain_wait(&bars[B_KFULL + st], (uint32_t)((k_iss[st] - 1) & 1));
        for (int st = 0; st < kVStages; ++st)
          if (v_iss[st] > 0) drain_wait(&bars[B_VFULL + st], (uint32_t)((v_iss[st] - 1) & 1));
      }
    }
  } else if (warp == 1) {
    // ================= retrieval and P V issuer =================
    // The whole warp runs the issue loop (waits, ring positions, descriptors), so
    // every value is warp-uniform, and one elected lane issues the tensor-core
    // operations and commits: issuing from a diverged single thread was several
    // times slower while the softmax warps on the same scheduler were busy. The
    // Q K^T products come from warp 10 on another scheduler, so each issuing warp
    // has half of the per-key-tile instruction stream. Shared-memory descriptors are
    // built once per buffer and moved by a constant add (a descriptor holds the
    // address / 16 in its low 14 bits and every operand lies below 256 KB, so an
    // offset inside a buffer never carries out of that field).
    {
      const uint32_t id_pv = idesc_f32acc(1, 0, 1, BM, D);
      const uint64_t dV0 = mnmajor_desc(smem_u32(sV), 0);
      constexpr uint32_t kTileD = kTile >> 4;  // one tile, in descriptor units
      uint32_t vst = 0, vph = 0;  // V ring: stage and phase of the next item
      uint32_t pn = 0;            // P products issued so far: P n sits in S buffer n & 1
      int tc = 0;
      auto v_next = [&]() {
        if (++vst == (uint32_t)kVStages) {
          vst = 0;
          vph ^= 1u;
        }
      };
      bool ok = true;
      for (;;) {
        // sigma(Q) of tile tc (or the softmax warps' end-of-list arrival) also orders
        // this read of its descriptor after the producer's write
        if (!mbar_wait_warp(&bars[B_SQFULL], (uint32_t)(tc & 1))) {
          ok = false;
          break;
        }
        const Tile t = slots[tc & 1];
        if (!t.valid) break;
        // retrieval: R = sigma(Q) M_hi, sigma(Q) read from tensor memory (features
        // 0..63 at O + [0, 32), features 64..127 at O + [64, 96))
        const uint32_t s0 = vst, p0 = vph;
        v_next();
        ok = mbar_wait_warp(&bars[B_VFULL + s0], p0);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dm0 = dV0 + s0 * kTileD;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16_ts(tR, tO + (kk < 4 ? 8 * kk : 64 + 8 * (kk - 4)), dm0 + mndesc_off(kk), id_pv,
                        kk > 0 ? 1u : 0u);
          mma_commit(&bars[B_VEMPTY + s0]);
          mma_commit(&bars[B_RDONE]);
        }
        __syncwarp();
        for (int j = 0; ok && j < t.nkv; ++j) {
          const uint32_t st = vst, ph = vph;
          v_next();
          const uint32_t pb = pn & 1u;
          ok = mbar_wait_warp(&bars[B_PFULL + pb], (pn >> 1) & 1u) &&
               mbar_wait_warp(&bars[B_VFULL + st], ph);
          if (!ok) break;
          tc_fence_after();
          // P_j lives in the first 64 columns of its S buffer
          const uint32_t tP = tS + pb * BN;
          const uint64_t dv = dV0 + st * kTileD;
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk)
              mma_bf16_ts(tO, tP + 8 * kk, dv + mndesc_off(kk), id_pv, (j > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&bars[B_VEMPTY + st]);
            // P V done: the S buffer may take the next Q K^T, and O may be rescaled
            mma_commit(&bars[B_SFREE + pb]);
          }
          __syncwarp();
          ++pn;
        }
        if (!ok) break;
        ++tc;
      }
      // no MMA may still be running when the CTA frees tensor memory
      if (elect_one()) mma_commit(&bars[B_DRAIN]);
      __syncwarp();
      drain_wait(&bars[B_DRAIN], 0);
    }
  } else if (warp == 2 + kSoftmaxWarps) {
    // ================= Q K^T issuer (warp 10) =================
    // Key step n (counted over the CTA's whole tile sequence) uses K stage and S
    // buffer n & 1. Its product overwrites the S buffer that held P of step n - 2,
    // so it waits for that step's P V (the S-free barrier of the buffer, committed by
    // warp 1); each S-free barrier completes once per use of its buffer and cannot
    // run two phases ahead of this warp, whose product the next P V needs.
    {
      const uint32_t id_qk = idesc_f32acc(1, 0, 0, BM, BN);
      const uint64_t dQ = kmajor_desc(smem_u32(sQ), 0);
      const uint64_t dK0 = kmajor_desc(smem_u32(sK), 0);
      constexpr uint32_t kTileD = kTile >> 4;
      uint32_t kst = 0, kph = 0;  // K stage / S buffer of the next step, and its use parity
      uint32_t n = 0;
      int tc = 0;
      bool ok = true;
      for (;;) {
        if (!mbar_wait_warp(&bars[B_QFULL], (uint32_t)(tc & 1))) {
          ok = false;
          break;
        }
        const Tile t = slots[tc & 1];
        if (!t.valid) break;
        for (int j = 0; j < t.nkv; ++j) {
          ok = (n < 2 || mbar_wait_warp(&bars[B_SFREE + kst], kph ^ 1u)) &&
               mbar_wait_warp(&bars[B_KFULL + kst], kph);
          if (!ok) break;
          tc_fence_after();
          const uint64_t dk = dK0 + kst * kTileD;
          const uint32_t dS = tS + kst * BN;
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_bf16_ss(dS, dQ + kdesc_off(kk), dk + kdesc_off(kk), id_qk, kk > 0 ? 1u : 0u);
            mma_commit(&bars[B_SFULL + kst]);  // also frees the K stage
            if (j == t.nkv - 1) mma_commit(&bars[B_QEMPTY]);
          }
          __syncwarp();
          kph ^= kst;
          kst ^= 1u;
          ++n;
        }
        if (!ok) break;
        ++tc;
      }
      if (elect_one()) mma_commit(&bars[B_DRAIN]);
      __syncwarp();
      drain_wait(&bars[B_DRAIN], 0);
    }
  } else {
    // ================= softmax / epilogue (warps 2..9) =================
    const int wq = warp & 3;
    const int half = (warp - 2) >> 2;  // key / value columns [64 half, 64 half + 64)
    const int r = wq * 32 + lane;      // query row inside the tile == tensor-memory lane
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t col0 = (uint32_t)half * 64;
    uint64_t* pair = &bars[B_PAIR + wq];  // the two warps that share these rows
    uint32_t pair_phase = 0;
    float* xmax = sX;            // [2 slots][2 halves][128]
    float* xden = sX + 512;      // [2 halves][128]
    float* xl = sX + 768;        // [2 halves][128]
    const float sl = 1.4426950408889634f * 0.08838834764831845f;  // log2(e) / sqrt(128)
    volatile int* sflag = reinterpret_cast<volatile int*>(smem + OFF_FLAG);
    long long kc = 0;
    int tc = 0;
    int sc = 0;  // split tiles met so far (phase of the split barriers)
    bool ok = true;
    // sigma(Q) of tile number tile_no (this thread's 64 columns) -> tensor memory
    // (O + 64 half, 32 packed columns) for the retrieval MMA; partial denominator
    // sigma(Q_r) . z_{s-1} over those columns.
    // the next tile's descriptor, after Q's full barrier: 1 a tile, 0 the end of the
    // list (arrive on sigma(Q)'s barrier once more so the P V warp sees it too),
    // -1 the wait gave up
    auto fetch = [&](int tile_no, Tile& tt) -> int {
      if (!mbar_wait_warp(&bars[B_QFULL], (uint32_t)(tile_no & 1))) return -1;
      tt = slots[tile_no & 1];
      if (tt.valid) return 1;
      mbar_arrive_warp(&bars[B_SQFULL]);
      return 0;
    };
    auto sigma_q = [&](int tile_no, float& den) -> bool {
      const float* zs = sZ + col0;
      float dp[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t sq[32];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t off = (uint32_t)half * kSub + sw128(r, u);
        const uint4 raw = *reinterpret_cast<const uint4*>(sQ + off);
        const float4 z0 = *reinterpret_cast<const float4*>(zs + u * 8);
        const float4 z1 = *reinterpret_cast<const float4*>(zs + u * 8 + 4);
        const float zz[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h[e]);
          const float p0 = elu1(f.x), p1 = elu1(f.y);
          dp[e] = fmaf(p0, zz[2 * e], dp[e]);
          dp[e] = fmaf(p1, zz[2 * e + 1], dp[e]);
          sq[4 * u + e] = pack_bf16x2(p0, p1);
        }
      }
      den = (dp[0] + dp[1]) + (dp[2] + dp[3]);
      mbar_arrive_warp(&bars[B_QEMPTY]);  // this warp is done reading Q
      tmem_st32_(tO + lane_off + 64 * half, sq);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive_warp(&bars[B_SQFULL]);
      return true;
    };
    Tile t, tn;
    float den = 0.f;
    int oc = 0;  // tiles stored through shared memory so far
    const int got = fetch(0, t);
    ok = got >= 0;
    bool have = got == 1;
    if (have) ok = sigma_q(0, den);
    while (ok && have) {
      const float bta = __ldg(beta + t.h);  // used in the epilogue
      float m_use = -INFINITY, l = 0.f;
      for (int j = 0; j < t.nkv; ++j) {
        const int b = (int)(kc & 1);
        if (!mbar_wait_warp(&bars[B_SFULL + b], (uint32_t)((kc >> 1) & 1))) {
          ok = false;
          break;
        }
        ++kc;
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld32(tS + lane_off + b * BN + col0, *reinterpret_cast<uint32_t(*)[32]>(sr));
        tmem_ld32(tS + lane_off + b * BN + col0 + 32,
                  *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
        tmem_wait_ld();
        if ((kSplit ? t.j0 : 0) + j == t.i) {  // the diagonal key tile: causal mask
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if ((int)col0 + c > r) sr[c] = __float_as_uint(-INFINITY);
        }
        float mx[8];
#pragma unroll
        for (int q8 = 0; q8 < 8; ++q8) {
          const float* v = reinterpret_cast<const float*>(sr);
          mx[q8] = fmax3(v[q8], v[8 + q8], v[16 + q8]);
          mx[q8] = fmax3(mx[q8], v[24 + q8], v[32 + q8]);
          mx[q8] = fmax3(mx[q8], v[40 + q8], v[48 + q8]);
          mx[q8] = fmaxf(mx[q8], v[56 + q8]);
        }
        const float mh = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                               fmaxf(mx[6], mx[7]));
        xmax[b * 256 + half * 128 + r] = mh;
        mbar_arrive_warp(pair);
        if (!mbar_wait_warp(pair, pair_phase & 1)) {
          ok = false;
          break;
        }
        ++pair_phase;
        const float mt = fmaxf(mh, xmax[b * 256 + (1 - half) * 128 + r]);
        bool need = false;
        float alpha = 1.f;
        if (j == 0) {
          m_use = mt;
        } else if ((mt - m_use) * sl > 8.f) {
          need = true;
          alpha = ex2_approx((m_use - mt) * sl);
          m_use = mt;
        }
        const float mb = m_use * sl;
        const uint64_t sl2 = f2pack(sl, sl), nmb2 = f2pack(-mb, -mb);
        uint64_t rsum2[2] = {f2pack(0.f, 0.f), f2pack(0.f, 0.f)};
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          float a0, a1, p0, p1;
          f2unpack(fma2(f2pack(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), sl2,
                        nmb2),
                   a0, a1);
          if ((c & 3) == 3) {
            ex2_poly2(a0, a1, p0, p1);
          } else {
            p0 = ex2_approx(a0);
            p1 = ex2_approx(a1);
          }
          rsum2[c & 1] = add2(rsum2[c & 1], f2pack(p0, p1));
          pk[c] = pack_bf16x2(p0, p1);
        }
        float r0, r1, r2, r3;
        f2unpack(rsum2[0], r0, r1);
        f2unpack(rsum2[1], r2, r3);
        const float rs = (r0 + r1) + (r2 + r3);
        // A rescale of O must wait for the previous step's P V (the S-free barrier of
        // its buffer). Only then: without a rescale nothing here touches O. The wait
        // cannot be misread: the barrier's previous phase completed before this
        // step's Q K^T was issued, and its next needs a P these warps have not written.
        const bool rescale = __any_sync(0xffffffffu, need);
        if (rescale && j > 0 &&
            !mbar_wait_warp(&bars[B_SFREE + ((kc - 2) & 1)], (uint32_t)(((kc - 2) >> 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (rescale) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + lane_off + col0 + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tO + lane_off + col0 + c * 32, o);
          }
          tmem_wait_st();
        }
        l = l * alpha + rs;
        // P (bf16) over the first 64 columns of this S buffer: half h at [32h, 32h + 32).
        // Both halves of every row have read their S values (the max exchange above).
        tmem_st32_(tS + lane_off + b * BN + 32 * half, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive_warp(&bars[B_PFULL + b]);
      }
      if (!ok) break;

      // ---- epilogue: out = (1 - g) O / l + g R / den ----
      // The row sum and denominator halves do not depend on the MMAs: exchange
      // them first. Then O and R become packed outputs in registers, the next
      // tile's sigma(Q) goes into O (the retrieval MMA waits for it), and the
      // global stores of this tile come last, overlapping the next tile's MMAs.
      xden[half * 128 + r] = den;
      xl[half * 128 + r] = l;
      mbar_arrive_warp(pair);
      if (!mbar_wait_warp(pair, pair_phase & 1)) {
        ok = false;
        break;
      }
      ++pair_phase;
      const float g = 1.f / (1.f + expf(-bta));
      const float den_t = den + xden[(1 - half) * 128 + r];
      const float l_t = l + xl[(1 - half) * 128 + r];
      const float gr = den_t != 0.f ? g / den_t : 0.f;
      if (!mbar_wait_warp(&bars[B_SFREE + ((kc - 1) & 1)], (uint32_t)(((kc - 1) >> 1) & 1)) ||
          !mbar_wait_warp(&bars[B_RDONE], (uint32_t)(tc & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // Split mode: every piece of a tile leaves its record (O against its reference
      // max m_use, and the row sum); the piece that finishes last merges the records
      // in piece order (the same sums whichever piece it is) and writes the output.
      bool emit = true;
      float mx = m_use, l_out = l_t;
      const float* recs = p.rec + (size_t)t.tid * p.Pmax * kRecFloats;
      if (kSplit && t.np > 1) {
        float* rec = p.rec + ((size_t)t.tid * p.Pmax + t.pc) * kRecFloats;
        float4* recO = reinterpret_cast<float4*>(rec);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + col0 + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 8; ++q)
            __stcg(recO + (half * 16 + c * 8 + q) * 128 + r,
                   make_float4(__uint_as_float(o[4 * q]), __uint_as_float(o[4 * q + 1]),
                               __uint_as_float(o[4 * q + 2]), __uint_as_float(o[4 * q + 3])));
        }
        if (half == 0) {
          __stcg(rec + kRecO + r, m_use);
          __stcg(rec + kRecO + 128 + r, l_t);
        }
        __threadfence();  // the record is visible device-wide before the count
        mbar_arrive_warp(&bars[B_SPLW]);
        if (warp == 2) {
          ok = mbar_wait_warp(&bars[B_SPLW], (uint32_t)(sc & 1));
          if (ok && lane == 0) {
            const unsigned done = atomicAdd(p.tile_ctr + t.tid, 1u);
            *sflag = done == (unsigned)t.np - 1u ? 1 : 0;
            __threadfence();
            mbar_arrive(&bars[B_SPLF]);
          }
          __syncwarp();
        }
        if (!ok || !mbar_wait_warp(&bars[B_SPLF], (uint32_t)(sc & 1))) {
          ok = false;
          break;
        }
        ++sc;
        emit = *sflag != 0;
        if (emit) {
          __threadfence();  // the other pieces' records, counted before this piece's
          for (int q = 0; q < t.np; ++q)
            if (q != t.pc) mx = fmaxf(mx, __ldcg(recs + q * kRecFloats + kRecO + r));
          l_out = 0.f;
          for (int q = 0; q < t.np; ++q) {
            const float mq = q == t.pc ? m_use : __ldcg(recs + q * kRecFloats + kRecO + r);
            const float lq = q == t.pc ? l_t : __ldcg(recs + q * kRecFloats + kRecO + 128 + r);
            l_out = fmaf(ex2_approx((mq - mx) * sl), lq, l_out);
          }
        }
      }
      const float go = (1.f - g) / l_out;
      uint32_t w[32];  // this row's 64 outputs, bf16 pairs
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        if (!emit) break;
        uint32_t o[32];
        if (kSplit && t.np > 1) {  // the merged O: sum over the pieces in piece order, each scaled to mx
          float acc[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) acc[e] = 0.f;
          for (int q = 0; q < t.np; ++q) {
            if (q == t.pc) {
              tmem_ld32(tO + lane_off + col0 + c * 32, o);
              tmem_wait_ld();
              const float a = ex2_approx((m_use - mx) * sl);
#pragma unroll
              for (int e = 0; e < 32; ++e) acc[e] = fmaf(a, __uint_as_float(o[e]), acc[e]);
            } else {
              const float* rq = recs + q * kRecFloats;
              const float a = ex2_approx((__ldcg(rq + kRecO + r) - mx) * sl);
              const float4* oq = reinterpret_cast<const float4*>(rq) + (half * 16 + c * 8) * 128 + r;
#pragma unroll
              for (int qq = 0; qq < 8; ++qq) {
                const float4 v4 = __ldcg(oq + qq * 128);
                acc[4 * qq] = fmaf(a, v4.x, acc[4 * qq]);
                acc[4 * qq + 1] = fmaf(a, v4.y, acc[4 * qq + 1]);
                acc[4 * qq + 2] = fmaf(a, v4.z, acc[4 * qq + 2]);
                acc[4 * qq + 3] = fmaf(a, v4.w, acc[4 * qq + 3]);
              }
            }
          }
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(acc[e]);
        } else {
          tmem_ld32(tO + lane_off + col0 + c * 32, o);
          tmem_wait_ld();
        }
        uint32_t rr[32];
        tmem_ld32(tR + lane_off + col0 + c * 32, rr);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float a0 = go * __uint_as_float(o[2 * e]) + gr * __uint_as_float(rr[2 * e]);
          const float a1 = go * __uint_as_float(o[2 * e + 1]) + gr * __uint_as_float(rr[2 * e + 1]);
          w[16 * c + e] = pack_bf16x2(a0, a1);
        }
      }
      tc_fence_before();
      // A whole tile (or one whose missing rows lie past the end of the tensor, where
      // TMA drops them) leaves through shared memory: each half writes its 128 x 64
      // box, 128B-swizzled, and the half's first warp issues the TMA store. Before a
      // half rewrites its box, that warp has seen its previous store finish reading.
      const bool tma_tile = emit && p.tma_out &&
                            (t.rows_valid == BM || (long long)t.q_row + t.rows_valid == p.L);
      const bool issuer = warp == 2 + 4 * half;
      if (tma_tile) {
        if (oc > 0) {
          if (issuer && lane == 0) {
            bulk_wait_group_read0();
            mbar_arrive(&bars[B_OFREE + half]);
          }
          __syncwarp();
          if (!mbar_wait_warp(&bars[B_OFREE + half], (uint32_t)((oc - 1) & 1))) {
            ok = false;
            break;
          }
        }
        const uint32_t ob = smem_u32(sOut + half * kSub);
#pragma unroll
        for (int u = 0; u < 8; ++u)
          st_shared_v4(ob + sw128(r, u), w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        fence_proxy_async_smem();
        mbar_arrive_warp(&bars[B_OFULL + half]);
        if (issuer) {
          if (!mbar_wait_warp(&bars[B_OFULL + half], (uint32_t)(oc & 1))) {
            ok = false;
            break;
          }
          if (lane == 0) {
            tma_store_4d(&tm_o, sOut + half * kSub, 64 * half, t.q_row, t.h, t.b);
            tma_store_commit();
          }
          __syncwarp();
        }
        ++oc;
      }
      const int gn = fetch(tc + 1, tn);
      const bool has_next = gn == 1;
      if (gn < 0 || (has_next && !sigma_q(tc + 1, den))) {
        ok = false;
        break;
      }
      if (emit && !tma_tile && r < t.rows_valid) {
        __nv_bfloat16* orow = out + t.b * p.o_sb + t.h * p.o_sh + (t.q_row + r) * p.o_sl + col0;
        if (p.out32) {
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) st_global_v8(orow + q8 * 16, w + 8 * q8);
        } else {
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            *reinterpret_cast<uint4*>(orow + q4 * 8) =
                make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
        }
      }
      t = tn;
      have = has_next;
      ++tc;
    }
    // the TMA stores must be done with shared memory (and global) before the CTA ends
    if (warp == 2 + 4 * half && lane == 0) tma_store_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t bf16_attn_set_attributes() {
  const cudaError_t e = cudaFuncSetAttribute(attn_kernel<false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(attn_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kAttnSmem);
}

namespace {
int split_tiles(int T, int C) {  // sum over tiles i < T of ceil((i + 1) / C)
  int n = 0;
  for (int i = 0; i < T; ++i) n += (i + C) / C;
  return n;
}
size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }
}  // namespace

Bf16AttnSplit bf16_attn_split_plan(int BH, int S, int N, long long L, int sms) {
  Bf16AttnSplit sp;
  if (L <= 0 || BH < 1 || S < 1) return sp;
  const int T = (int)((min((long long)N, L) + BM - 1) / BM);
  const long long pairs = (long long)BH * S * ((T + 1) / 2);
  if (pairs >= sms) return sp;
  // Fewer pairs than SMs: whole query tiles, heaviest first, one per CTA as far as they
  // go (no records, no merge) while there are at least half as many tiles as SMs.
  // Fewer tiles than that: pieces, the longest that still give about 1.25 units per
  // SM (a longer piece spends less on its prologue, record and merge), at least
  // ceil(T / 8) key tiles each.
  if ((long long)BH * S * T * 2 >= sms) {
    sp.C = T;
    sp.Pmax = 1;
    sp.units = (long long)BH * S * T;
    return sp;
  }
  const int cmin = max(1, (T + 7) / 8);
  int C = cmin;
  for (int c = T; c >= cmin; --c)
    if ((long long)BH * S * split_tiles(T, c) * 4 >= 5LL * sms) {
      C = c;
      break;
    }
  sp.C = C;
  sp.Pmax = (T + C - 1) / C;
  sp.units = (long long)BH * S * split_tiles(T, C);
  return sp;
}

size_t bf16_attn_split_bytes(const Bf16AttnSplit& sp, int BH, int S, int N, long long L) {
  if (sp.C == 0) return 0;
  const int T = (int)((min((long long)N, L) + BM - 1) / BM);
  const size_t tiles = (size_t)BH * S * T;
  // whole tiles (Pmax 1) leave no records
  return 256 + up256(tiles * 4) + (sp.Pmax > 1 ? tiles * sp.Pmax * kRecFloats * sizeof(float) : 0);
}

cudaError_t bf16_attn_launch(const __nv_bfloat16* q, const __nv_bfloat16* k,
                             const __nv_bfloat16* v, const float* beta, __nv_bfloat16* out,
                             const Bf16Workspace& ws, int BH, int H, long long L, int N, int S,
                             cudaStream_t stream, const Bf16Layout* lay,
                             const Bf16AttnSplit* split, void* split_ws) {
  // query head (b, h) reads key/value head (b, h / (H / H_kv)); out is laid out as q
  const Bf16Layout l = lay ? *lay : Bf16Layout::bhld(BH / H, H, L);
  if ((long long)l.B * l.H != BH || l.H_kv < 1 || l.H % l.H_kv != 0) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv, mm, mo;
  if (!make_bf16_map4(&mq, q, (uint64_t)L, l.H, l.B, l.q_sl, l.q_sh, l.q_sb, 128) ||
      !make_bf16_map4(&mk, k, (uint64_t)L, l.H_kv, l.B, l.kv_sl, l.kv_sh, l.kv_sb, 128) ||
      !make_bf16_map4(&mv, v, (uint64_t)L, l.H_kv, l.B, l.kv_sl, l.kv_sh, l.kv_sb, 128) ||
      !make_bf16_map(&mm, ws.Mhl, D, (uint64_t)l.B * l.H_kv * S * 2, 128))
    return cudaErrorInvalidValue;
  Params p{};
  p.L = L;
  p.N = N;
  p.S = S;
  p.H = l.H;
  p.Hkv = l.H_kv;
  p.BH = BH;
  p.o_sb = l.q_sb;
  p.o_sh = l.q_sh;
  p.o_sl = l.q_sl;
  p.T = (int)((min((long long)N, L) + BM - 1) / BM);
  p.U = (p.T + 1) / 2;
  long long units = (long long)BH * S * p.U;
  if (split && split->C > 0 && split_ws) {
    // counters first (zeroed here, on the launch stream), then the records
    const size_t tiles = (size_t)BH * S * p.T;
    if (cudaMemsetAsync(split_ws, 0, 256 + up256(tiles * 4), stream) != cudaSuccess)
      return cudaErrorInvalidValue;
    p.split = 1;
    p.C = split->C;
    p.Pmax = split->Pmax;
    p.BHS = (unsigned)(BH * S);
    p.divBHS = FastDiv(p.BHS);
    p.unit_ctr = static_cast<unsigned*>(split_ws);
    p.tile_ctr = reinterpret_cast<unsigned*>(static_cast<char*>(split_ws) + 256);
    p.rec = reinterpret_cast<float*>(static_cast<char*>(split_ws) + 256 + up256(tiles * 4));
    units = split->units;
  }
  if (units >= (1ll << 31)) return cudaErrorInvalidValue;
  p.units = (unsigned)units;
  p.divU = FastDiv((uint32_t)p.U);
  p.divS = FastDiv((uint32_t)S);
  p.divH = FastDiv((uint32_t)l.H);
  p.divG = FastDiv((uint32_t)(l.H / l.H_kv));
  p.out32 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0 ? 1 : 0;
  // a TMA map needs a 16-byte aligned base; otherwise every tile is stored directly
  p.tma_out = make_bf16_map4(&mo, out, (uint64_t)L, l.H, l.B, l.q_sl, l.q_sh, l.q_sb, 128) ? 1 : 0;
  if (!p.tma_out) mo = mq;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const unsigned grid = p.units < (unsigned)sms ? p.units : (unsigned)sms;
  if (grid == 0) return cudaSuccess;
  if (p.split)
    attn_kernel<true><<<grid, kThreads, kAttnSmem, stream>>>(mq, mk, mv, mm, mo, beta, ws.zprev,
                                                             out, p);
  else
    attn_kernel<false><<<grid, kThreads, kAttnSmem, stream>>>(mq, mk, mv, mm, mo, beta, ws.zprev,
                                                              out, p);
  return cudaGetLastError();
}

}  // namespace infini
