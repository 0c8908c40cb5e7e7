// fwd_common.cuh -- shared definitions of the prefill kernel (gptoss_attn_fwd).
//
// Rule: GptOssAttention on the NeMo AutoModel gpt_oss.layers page (sinks,
// sliding_window, softmax_scale = head_dim^-0.5, grouped query heads), RoPE of
// the gpt_oss.rope_utils page, sink in the denominator only (Transformers
// v4.55.0 release notes, "Architecture").
//
// Design: persistent CTAs (one per SM), each walking a static, heaviest-first
// list of work units.  A unit is one 128-query tile of TWO query heads that
// share a kv head, so every K/V tile is loaded once for 256 query rows.
// 16 warps (roles in fwd_softmax.cuh, fwd_rope.cuh, fwd_pipeline.cuh):
//   warps 0-3         rope: the Q tiles (and, without a workspace, the K
//                     tiles) rotated in place after TMA
//   warps 4-7 / 8-11  softmax of head A / head B (thread = query row; warp w
//                     reads TMEM lanes 32 (w % 4) .. 32 (w % 4) + 31)
//   warp 12           TMA producer of the K / V tiles (4-stage ring)
//   warp 13           TMEM allocation; QK^T issue (fwd_mma_s_role)
//   warp 14           P V issue (fwd_mma_pv_role)
//   warp 15           TMA producer of the Q tiles (two per unit, 3-stage
//                     ring: a unit's Q arrives while the two before it run)
// setmaxnreg moves registers from the rope / producer / MMA warpgroups to the
// two softmax warpgroups: launch 512 threads x 128 registers = 65536, split
// 2 x 128 x 208 + 128 x 48 + 128 x 48 = 65536.  The host refuses to launch if
// the compiled kernel does not start at exactly 128 registers per thread.
// TMEM columns (all 512): S_A [0,128) P_A [128,192) O_A [192,256),
//                         S_B [256,384) P_B [384,448) O_B [448,512).
#pragma once

#include "host_util.cuh"
#include "rope_qk.cuh"
#include "sm100_ptx.cuh"

namespace gptoss {

constexpr int kFwdTile = 128;         // query rows and keys per tile
constexpr int kFwdStages = 3;         // K / V ring (measured: 3 stages beat 4 by 2-4 %)
constexpr int kFwdQStages = 3;        // Q ring (units)
constexpr int kFwdThreads = 512;
constexpr int kFwdLaunchRegs = 128;   // 65536 / 512
constexpr int kFwdTileBytes = kFwdTile * kHeadDim * 2;  // 16 KB
constexpr uint32_t kFwdTmemCols = 512;
// Tensor memory, two layouts.  Three S buffers (the causal-only kernel at
// D = 64, and D = 128): three 128-column S buffers at 128 b (P, fp16, is
// written over the first 64 columns of the S it came from), then O from
// column 384 (64 columns per head slot at D = 64, 128 at D = 128); score
// products k = 0, 1, 2, .. (tile t of head slot X is k = t * slots + X) take
// buffer k mod 3, whose previous product's P V must have completed first.
// Per slot (the sliding-window kernel at D = 64): S_X at 256 X, P_X at
// 256 X + 128, O_X at 256 X + 192; the next S of a slot is issued as soon
// as its softmax has read the current one.  (Measured: the three-buffer
// layout takes full causal from 1.86 to 1.57 ms but the sliding window from
// 202 to 225 us, whose two-tile units then wait for a P V before each S.)
constexpr int kSBufs = 3;
constexpr uint32_t kColO = 384;
// A row's base moves when a tile's maximum exceeds it by more than this (log2
// units): P = 2^(s - base) then stays at or below 2^15, inside fp16's range.
constexpr float kRescaleThreshold = 15.0f;
constexpr uint32_t kRegsSoftmax = 208, kRegsRope = 48, kRegsOther = 48;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsRope + 128 * kRegsOther == kFwdThreads * kFwdLaunchRegs,
              "register split must add up to the launch allocation");

struct FwdParams {
  CUtensorMap tmap_q;  // dims (64, Hq, S or T, B or 1), box (64, 1, 128, 1)
  CUtensorMap tmap_k;  // fp16 k of the workspace, dims (64, Hkv, S or T, B or 1), box (64, 1, 128, 1)
  CUtensorMap tmap_v;  // fp16 v of the workspace, same layout
  const __nv_bfloat16* q;
  gptoss_strides sq;
  __nv_bfloat16* out;
  gptoss_strides so;
  float* lse;
  const float* sinks;         // nullable: no sink (the block form; the merge folds it in)
  const int32_t* positions;
  const int32_t* cu_seqlens;
  int B, S, T, Hq, Hkv, G, HP, window, n_qtiles, n_units;
  // Block form (BSHD): the keys are another block of the sequence than the
  // queries.  Query row i and key row j sit at global indices i + delta and
  // j (delta = first query's global index - first key's, >= 0); Lk keys per
  // batch row.  Self-attention: delta = 0, Lk = S.
  int delta, Lk;
  float* out_f32;             // nullable: fp32 output [B, S, Hq, 64] dense instead of bf16 out
  const float2* cs_tab;  // nullable: per-token (c cos, c sin) of the 32 pairs, [token][32]
  float scale_log2;
  uint64_t wait_ns;
  RopeTable tab;
};

struct __align__(1024) FwdSmem {
  uint8_t q[kFwdQStages][2][kFwdTileBytes];  // [stage][head A/B], rotated, 128B-swizzled
  uint8_t k[kFwdStages][kFwdTileBytes];
  uint8_t v[kFwdStages][kFwdTileBytes];
  uint64_t q_loaded[kFwdQStages], q_full[kFwdQStages], q_empty[kFwdQStages];  // TMA landed / rotated / free
  uint64_t k_full[kFwdStages], k_empty[kFwdStages];
  uint64_t v_full[kFwdStages], v_empty[kFwdStages];
  // Parity waits tell only adjacent phases apart, so every barrier is laid
  // out so that its waiter has seen the previous phase complete and the next
  // one cannot start before the waiter acts:
  //   s_full[X][b]: slot X's product landed in S buffer b (a slot uses each
  //     buffer once every three tiles, tile t being its use t / 3; per buffer
  //     alone, a slot could poll before the other slot's earlier product in
  //     that buffer had landed and take the old phase for its own);
  //   p_full[b]: the product's P is in buffer b (the P V issuer takes products
  //     in order; per slot, a slot's softmax could finish two tiles before
  //     the issuer looks);
  //   s_empty[b]: the P V that read buffer b's P completed.
  uint64_t s_full[2][kSBufs], p_full[kSBufs], s_empty[kSBufs];
  uint64_t o_done[2];  // per head slot A/B
  // per-slot layout: s_full[X][0] and p_full[X] serve slot X, and s_free[X]
  // tells the QK^T issuer that slot X's softmax has read its S
  uint64_t s_free[2];
  uint64_t mma_final[2];  // the S and P V issuers' last products have completed
  uint32_t tmem_base;
};

// One work unit: query tile q0 / 128 of heads (h0, h1) of sequence b.
struct Unit {
  int b, h0, h1, g, q0, L, Lk, seq_start, j_lo, n_kt;  // L query rows, Lk key rows
  bool dup;  // h1 repeats h0 (odd group size): computed, not stored
};

// Unit u of the static list (heaviest query tiles first).  Returns false for
// a tile past the end of its packed sequence; every role skips the same units.
// kPair: a unit holds two heads of a group (p.HP = ceil(G / 2) pairs);
// otherwise one (p.HP = G), h1 = h0 and nothing is duplicated.
template <bool kPair = true>
__device__ __forceinline__ bool make_unit(const FwdParams& p, int u, Unit& w) {
  const int per_tile = p.B * p.Hkv * p.HP;
  const int qt = p.n_qtiles - 1 - u / per_tile;
  int rest = u % per_tile;
  const int hp = rest % p.HP;
  rest /= p.HP;
  w.g = rest % p.Hkv;
  w.b = rest / p.Hkv;
  if (kPair) {
    w.h0 = w.g * p.G + 2 * hp;
    w.dup = (2 * hp + 1) >= p.G;
    w.h1 = w.dup ? w.h0 : w.h0 + 1;
  } else {
    w.h0 = w.h1 = w.g * p.G + hp;
    w.dup = false;
  }
  const bool thd = p.cu_seqlens != nullptr;
  w.seq_start = thd ? __ldg(p.cu_seqlens + w.b) : 0;
  w.L = thd ? __ldg(p.cu_seqlens + w.b + 1) - w.seq_start : p.S;
  // cu_seqlens: nondecreasing, within the T tokens, no sequence longer than S
  // (every role decodes the same unit, so all skip a bad one together)
  if (thd && !index_ok(w.seq_start >= 0 && w.L >= 0 && w.seq_start + w.L <= p.T && w.L <= p.S)) return false;
  w.Lk = thd ? w.L : p.Lk;
  w.q0 = qt * kFwdTile;
  if (w.q0 >= w.L) return false;
  // keys visible from the tile's rows: [q0 + delta - window + 1, q_last + delta]
  const int q_last = min(w.q0 + kFwdTile, w.L) - 1;
  const int j_hi = min(q_last + p.delta, w.Lk - 1) / kFwdTile;
  w.j_lo = p.window > 0 ? max(0, w.q0 + p.delta - p.window + 1) / kFwdTile : 0;
  w.n_kt = j_hi - w.j_lo + 1;
  return true;
}

// Byte offset of the 32-bit word holding features (e, e+1) of row r in a
// 128B-swizzled 128 x 64 bf16 tile (e even).
__device__ __forceinline__ uint32_t sw128_word(int r, int e) {
  return r * 128 + ((((e >> 3) ^ (r & 7))) << 4) + (e & 7) * 2;
}

// Rotates the two pairs held in bf16 words (lo, hi) = features (e, e+1),
// (e+32, e+33) and returns them as fp16: the rotated q / k feed the QK^T
// product in fp16, whose 11-bit significand leaves eight times less rounding
// in the concentration-scaled logits than bf16 would (the rotated values must
// stay inside the fp16 range, |x| < 65504; GPT-OSS activations are O(10)).
__device__ __forceinline__ void rotate_words(uint32_t& lo, uint32_t& hi, float2 a, float2 b) {
  const float x0 = bf16lo(lo), x1 = bf16hi(lo);
  const float y0 = bf16lo(hi), y1 = bf16hi(hi);
  lo = pack_f16(x0 * a.x - y0 * a.y, x1 * b.x - y1 * b.y);
  hi = pack_f16(y0 * a.x + x0 * a.y, y1 * b.x + x1 * b.y);
}

// (c, s) * (cos d, sin d): advances an angle seed by a fixed step.
__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
  return make_float2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}

template <uint32_t N>
__device__ __forceinline__ void reg_alloc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void reg_dealloc() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

}  // namespace gptoss
