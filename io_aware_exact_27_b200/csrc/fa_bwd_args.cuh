// Arguments and workspace layout shared by the backward kernels (the
// preparation of D and LSE, the dK/dV and dQ kernels, the block-sparse work
// lists).
#pragma once

#include "fa_common.cuh"

namespace fa {

constexpr int kThreadsBwd = 320;  // 8 elementwise warps, producer, MMA issuer
constexpr int kVecSlack = 128;    // workspace rows past the last token of each head
constexpr float kLog2e = 1.4426950408889634f;

struct BwdArgs {
  const void* o;
  const void* dout;
  const float* lse;     // forward LSE (natural log)
  void* dq;
  void* dk;
  void* dv;
  float* lse2;          // workspace [Hq][ws_stride]: LSE * log2(e), +inf where no token
  float* dvec;          // workspace [Hq][ws_stride]: D, 0 where no token
  const int* cu_seqlens;
  int nseq;             // padded: B
  int N;                // padded: N; varlen: max_seqlen
  int total_T;
  int Hq, Hkv;
  int causal;
  float scale;
  float scale_log2;
  int lse_head_stride;  // forward LSE: padded N, varlen total_T
  int ws_stride;        // round_up4(total_T) + 4 * nseq + 128 (see ws_offset)
  int num_units;
  uint64_t timeout_ns;
  int* status;
  // block-sparse: [Hq][nqb][nqb] uint8 as for the forward; null = dense
  const uint8_t* block_mask;
  int nqb;
  // block-sparse dK/dV work plan (written by fa_bwd_plan_kernel): plan[0] =
  // items, plan[1] = split units; from int 4 on, plan_max_items items of 4
  // ints (unit, first visible step, steps, partial slot or -1), then the
  // split units (unit, first slot, chunks, 0). partials: [slot][dV, dK]
  // [128 rows][D] fp32 sums of a split unit's chunks.
  int* plan;
  float* partials;
  int plan_max_items;
  int plan_max_slots;
  int* plan_nbuf;   // visible steps per unit
  int* plan_sbase;  // first entry of each unit's steps in plan_steps
  int* plan_steps;  // every unit's visible steps, in order (unit after unit)
  // block-sparse dQ: per row r = h * nqb + query tile, the visible key
  // blocks (causal: at or below the diagonal) in order at rows_list[rows_base[r]..]
  int* rows_n;
  int* rows_base;
  int* rows_list;
  // fp8 (the score products on e4m3 codes): block scales [B, H, nblk_s] of
  // the Q and K codes (value = code * scale); null for bf16
  const float* q_scale;
  const float* k_scale;
  int nblk_s;
};

// Workspace layout: per query head, sequence s's rows start at
//   ws_offset(s) = round_up(first token of s, 4) + 4 * s,
// a 16-byte aligned float offset, so that the 128-row vectors of a query
// tile can be fetched with one bulk copy; gaps and the 128 trailing entries
// per head hold +inf (LSE) and 0 (D), harmless when a tile runs past the end
// of its sequence.
__device__ __forceinline__ int ws_offset(int tok0, int seq) { return ((tok0 + 3) & ~3) + 4 * seq; }

}  // namespace fa
