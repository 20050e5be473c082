// Decode: a few new query rows per sequence against a long key/value cache
// (the KV-cache entry point of the Dao-AILab repository overview), split
// over the cache ("split-KV") so that small batches still fill the GPU,
// and the per-split results combined through their log-sum-exp.
//
// Query i of Nq sits at position L_b - Nq + i of sequence b (L_b valid
// cache rows); causal attention lets it see keys 0 .. L_b - Nq + i. A row
// that sees no key gets O = 0 and LSE = -inf.
//
// Work unit = (batch b, kv head, split): the R = Nq * (Hq/Hkv) <= 16 query
// rows that read that kv head, against one contiguous range of the cache.
// The query rows are too few for a 128-row MMA tile, so both products are
// taken transposed and the rows sit in the MMA's N = 16:
//   S^T [128 keys, 16 rows]  = K_j Q^T      (A = K tile, K-major, from TMA)
//   O^T [d, 16 rows]        += V_j^T P_j^T  (A = V tile read MN-major)
// with fp32 accumulators in TMEM. The path streams the cache once: it is
// bound by HBM, and the tensor cores only keep the CUDA cores free for the
// softmax. Warp roles of the persistent CTA (one per SM):
//   warps 0-7  softmax, two groups of four that take alternate tiles (the
//              per-tile chain of TMEM load, barrier, exponentials and P store
//              is latency-bound, so two tiles are kept in flight). Thread =
//              key of the tile (TMEM lane), 16 row columns; each group keeps
//              its own lazy running maximum (base 2, threshold 8), row sums
//              and O^T accumulator, and the unit's epilogue combines the two
//              exactly, as two key ranges are combined through their LSE.
//              P^T goes to shared memory as the bf16 B operand.
//   warp 8     TMA producer: Q rows of each unit, K/V tiles through a ring
//   warp 9     tcgen05.mma issuer
// fa_decode_merge_kernel combines the splits' (O_r, LSE_r):
//   LSE = log sum exp LSE_r,  O = sum exp(LSE_r - LSE) O_r.
#pragma once

#include "fa_common.cuh"

namespace fa {

constexpr int kDecRows = 16;   // N of both MMAs: max Nq * (Hq/Hkv)
constexpr int kDecKeys = 128;  // keys per tile (M of the score MMA)
constexpr int kDecWarpProducer = 8;
constexpr int kDecWarpMma = 9;
constexpr int kDecThreads = 320;
constexpr int kDecBarGroup = 1;    // named barriers 1, 2: the 4 warps of softmax group 0, 1
constexpr int kDecBarSoftmax = 3;  // named barrier of all 8 softmax warps
constexpr float kDecTau = 8.f;     // lazy-rescale threshold (log2 units)

struct DecArgs {
  const void* q;              // [B, Nq, Hq, d] bf16
  const int* cache_seqlens;   // [B] device
  void* o;                    // [B, Nq, Hq, d] bf16 (single split)
  float* lse;                 // [B, Hq, Nq] (single split)
  float* part_o;              // [splits][B][Nq][Hq][d] fp32 (several splits)
  float* part_lse;            // [splits][B][Hq][Nq]
  int B, Nq, Hq, Hkv, Ncache;
  int splits, chunk;          // keys per split (multiple of kDecKeys)
  int num_units;              // B * Hkv * splits
  int causal;
  float scale_log2;
  uint64_t timeout_ns;
  int* status;
};

template <int D>
struct DecSmem {
  static constexpr int kStages = D == 128 ? 3 : 6;
  static constexpr int kTileBytes = kDecKeys * D * 2;  // one K or V tile, D/64 boxes of 16 KB
  static constexpr int kRowBox = kDecRows * 128;       // 16 rows x 128 bytes
  alignas(1024) uint8_t kv[kStages][2][kTileBytes];    // [slot][K, V]
  alignas(1024) uint8_t q[2][D / 64][kRowBox];         // query rows of a unit, double-buffered
  alignas(1024) uint8_t p[2][2][kRowBox];              // P [16 rows, 128 keys] bf16 (two 64-key atoms), x2
  float red_m[2][kDecRows][4];                         // per group: per-warp column maxima
  float red_l[2][kDecRows][4];                         // per group: per-warp column sums
  float xm[2][2][kDecRows], xl[2][2][kDecRows];        // [unit parity][group]: running max, row sums
  int xn[2][2];                                        // [unit parity][group]: tiles the group took
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[2], s_free[2];
  uint64_t o_full[2], o_empty[2];
  uint64_t p_full[2];  // per softmax group (P buffer)
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

struct DecUnit {
  int b, hk, split, Lb, k_begin, k_end, ntiles;
};

__device__ __forceinline__ DecUnit dec_unit(const DecArgs& a, int u) {
  DecUnit w;
  w.split = u % a.splits;
  const int rest = u / a.splits;
  w.hk = rest % a.Hkv;
  w.b = rest / a.Hkv;
  w.Lb = min(max(__ldg(a.cache_seqlens + w.b), 0), a.Ncache);
  w.k_begin = w.split * a.chunk;
  w.k_end = min(w.Lb, w.k_begin + a.chunk);
  w.ntiles = w.k_end > w.k_begin ? (w.k_end - w.k_begin + kDecKeys - 1) / kDecKeys : 0;
  return w;
}

// Reduces 16 per-lane values over the 32 lanes of a warp, one column at a
// time, halving the columns each step: 16 shuffles in all. Afterwards lanes
// 2c and 2c+1 hold the result for column c = (lane >> 1) & 15.
template <bool MAX>
__device__ __forceinline__ float warp_colreduce16(const float (&v)[16], int lane) {
  auto op = [](float x, float y) { return MAX ? fmaxf(x, y) : x + y; };
  float a8[8], a4[4], a2[2];
  const bool h16 = lane & 16, h8 = lane & 8, h4 = lane & 4, h2 = lane & 2;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float send = h16 ? v[i] : v[i + 8];
    const float keep = h16 ? v[i + 8] : v[i];
    a8[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 16));
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float send = h8 ? a8[i] : a8[i + 4];
    const float keep = h8 ? a8[i + 4] : a8[i];
    a4[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 8));
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float send = h4 ? a4[i] : a4[i + 2];
    const float keep = h4 ? a4[i + 2] : a4[i];
    a2[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 4));
  }
  const float send = h2 ? a2[0] : a2[1];
  const float keep = h2 ? a2[1] : a2[0];
  const float a1 = op(keep, __shfl_xor_sync(0xffffffffu, send, 2));
  return op(a1, __shfl_xor_sync(0xffffffffu, a1, 1));
}

// Byte offset of P[r][key] in the K-major, 128-byte-swizzled B operand
// [16 rows, 128 keys]: keys 0-63 in the first 2 KB atom, 64-127 in the second.
__device__ __forceinline__ int dec_p_offset(int r, int key) {
  return (key >> 6) * (kDecRows * 128) + r * 128 + (((((key & 63) >> 3) ^ (r & 7))) << 4) + (key & 7) * 2;
}

// Writes O = 0 and LSE = -inf for the rows of a unit that has no visible key.
template <int D>
__device__ __forceinline__ void dec_write_empty(const DecArgs& a, const DecUnit& w, int tid, int G, int R) {
  for (int r = 0; r < R; ++r) {
    const int i = r / G, hq = w.hk * G + (r - i * G);
    const size_t orow = (static_cast<size_t>(w.b) * a.Nq + i) * a.Hq + hq;
    const size_t li = (static_cast<size_t>(w.b) * a.Hq + hq) * a.Nq + i;
    if (a.splits == 1) {
      if (tid < D) reinterpret_cast<__nv_bfloat16*>(a.o)[orow * D + tid] = __float2bfloat16_rn(0.f);
      if (tid == 0) a.lse[li] = -INFINITY;
    } else {
      const size_t ps = static_cast<size_t>(w.split) * a.B * a.Nq * a.Hq;
      if (tid < D) a.part_o[(ps + orow) * D + tid] = 0.f;
      if (tid == 0) a.part_lse[ps + li] = -INFINITY;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kDecThreads, 1)
    fa_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const DecArgs a) {
  using Smem = DecSmem<D>;
  constexpr int ST = Smem::kStages;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.Hq / a.Hkv;
  const int R = a.Nq * G;  // rows r = i*G + g  ->  query i, head hk*G + g

  if (tid == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(smem_u32(&sm.kv_full[s]), 1);
      mbar_init(smem_u32(&sm.kv_empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.q_full[i]), 1);
      mbar_init(smem_u32(&sm.q_empty[i]), 1);
      mbar_init(smem_u32(&sm.s_full[i]), 1);
      mbar_init(smem_u32(&sm.s_free[i]), 4);  // one arrival per softmax warp
      mbar_init(smem_u32(&sm.o_full[i]), 1);
      mbar_init(smem_u32(&sm.o_empty[i]), 8);  // every softmax warp reads both groups' O^T
    }
    for (int i = 0; i < 2; ++i) mbar_init(smem_u32(&sm.p_full[i]), 4);
    mbar_init(smem_u32(&sm.drain), 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  if (warp == kDecWarpMma) {
    tmem_alloc(smem_u32(&sm.tmem_base), 128);  // S^T per group, O^T per group x 2 units: 16 columns each
    tmem_relinquish();
  }
  if (warp == kDecWarpProducer && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const volatile int* abort = &sm.abort;
  uint32_t prod_issued = 0;  // K/V tiles issued by the producer thread
  uint32_t q_issued = 0;     // query-row loads issued by the producer thread

  if (warp == kDecWarpProducer) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      uint32_t kv_prod = 0, nu = 0;
      bool ok = true;
      DecUnit w_next = dec_unit(a, blockIdx.x);
      for (int u = blockIdx.x; u < a.num_units && ok; u += gridDim.x) {
        const DecUnit w = w_next;  // the next unit's cache length is loaded a unit ahead
        if (u + static_cast<int>(gridDim.x) < a.num_units) w_next = dec_unit(a, u + gridDim.x);
        if (w.ntiles == 0) continue;
        const uint32_t qb = nu & 1;
        if (!mbar_wait(smem_u32(&sm.q_empty[qb]), ((nu >> 1) & 1) ^ 1, abort, a.timeout_ns)) {
          report_error(a.status, kStatusTimeout, 90);
          ok = false;
          break;
        }
        const uint32_t qbar = smem_u32(&sm.q_full[qb]);
        mbar_expect_tx(qbar, static_cast<uint32_t>(R * 128 * (D / 64)));
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx)
          tma_load_3d(smem_u32(sm.q[qb][bx]), &tm_q, qbar, bx * 64, w.hk * G, w.b * a.Nq);
        q_issued = ++nu;
        const int row0 = w.b * a.Ncache + w.k_begin;  // first cache token of the unit
        for (int t = 0; t < w.ntiles; ++t) {
          const uint32_t slot = kv_prod % ST;
          if (!mbar_wait(smem_u32(&sm.kv_empty[slot]), ((kv_prod / ST) & 1) ^ 1, abort, a.timeout_ns)) {
            report_error(a.status, kStatusTimeout, 91);
            ok = false;
            break;
          }
          const uint32_t bar = smem_u32(&sm.kv_full[slot]);
          mbar_expect_tx(bar, 2 * Smem::kTileBytes);
#pragma unroll
          for (int bx = 0; bx < D / 64; ++bx) {
            tma_load_3d(smem_u32(sm.kv[slot][0]) + bx * 16384, &tm_k, bar, bx * 64, w.hk, row0 + t * kDecKeys);
            tma_load_3d(smem_u32(sm.kv[slot][1]) + bx * 16384, &tm_v, bar, bx * 64, w.hk, row0 + t * kDecKeys);
          }
          ++kv_prod;
        }
      }
      if (!ok) sm.abort = 1;
      prod_issued = kv_prod;
    }
  } else if (warp == kDecWarpMma) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kDecKeys, kDecRows, false, false);
      constexpr uint32_t idPV = idesc_bf16_f32(128, kDecRows, true, false);
      // V^T as an MN-major A of M = 128: the next 64 columns of d sit one
      // 16 KB box further; with d = 64 both halves of M read the same box
      // (TMEM lanes 64-127 then repeat lanes 0-63 and are not read).
      constexpr uint32_t kVLbo = D == 128 ? 16384 : 0;
      uint32_t kv_cons = 0, g = 0, nu = 0, npv = 0;
      bool ok = true;
      bool have_prev = false, prev_last = false;
      uint32_t prev_slot = 0, prev_nu = 0;
      int prev_t = 0;
      auto wait = [&](uint64_t* bar, uint32_t parity, int site) -> bool {
        if (!mbar_wait(smem_u32(bar), parity, abort, a.timeout_ns)) {
          report_error(a.status, kStatusTimeout, site);
          return false;
        }
        tc_fence_after();
        return true;
      };
      // O^T += V^T P^T for the previous tile, once its P is in shared memory
      auto issue_pv = [&]() -> bool {
        const uint32_t pb = npv & 1;  // P buffer of the tile
        if (!wait(&sm.p_full[pb], (npv >> 1) & 1, 92)) return false;
        const uint64_t pdesc = smem_desc(smem_u32(sm.p[pb]), 16, 1024, kSwizzle128B);
        const uint32_t ob = prev_nu & 1;
        if (prev_t == 0 && !wait(&sm.o_empty[ob], ((prev_nu >> 1) & 1) ^ 1, 93)) return false;
        const uint64_t vdesc = smem_desc(smem_u32(sm.kv[prev_slot][1]), kVLbo, 1024, kSwizzle128B);
        const uint32_t o_t = tmem + 32 + 32 * pb + 16 * ob;  // O^T of the tile's group
#pragma unroll
        for (int kk = 0; kk < kDecKeys / 16; ++kk)
          mma_f16_ss(o_t, vdesc + static_cast<uint64_t>((kk * 2048) >> 4),
                     pdesc + static_cast<uint64_t>(((kk >> 2) * 2048 + (kk & 3) * 32) >> 4), idPV,
                     (kk > 0 || prev_t >= 2) ? 1u : 0u);  // a group's first tile of the unit overwrites
        tc_commit(smem_u32(&sm.kv_empty[prev_slot]));
        if (prev_last) tc_commit(smem_u32(&sm.o_full[ob]));
        ++npv;
        return true;
      };
      DecUnit w_next = dec_unit(a, blockIdx.x);
      for (int u = blockIdx.x; u < a.num_units && ok; u += gridDim.x) {
        const DecUnit w = w_next;  // the next unit's cache length is loaded a unit ahead
        if (u + static_cast<int>(gridDim.x) < a.num_units) w_next = dec_unit(a, u + gridDim.x);
        if (w.ntiles == 0) continue;
        const uint32_t qb = nu & 1;
        if (!(ok = wait(&sm.q_full[qb], (nu >> 1) & 1, 94))) break;
        const uint64_t qdesc = smem_desc(smem_u32(sm.q[qb][0]), 16, 1024, kSwizzle128B);
        for (int t = 0; t < w.ntiles; ++t) {
          const uint32_t slot = kv_cons % ST;
          if (!(ok = wait(&sm.kv_full[slot], (kv_cons / ST) & 1, 95))) break;
          const uint32_t sb = g & 1;
          if (!(ok = wait(&sm.s_free[sb], ((g >> 1) & 1) ^ 1, 96))) break;
          // S^T = K_j Q^T: A = K tile (128 keys, K-major), B = query rows (16, K-major)
          const uint64_t kdesc = smem_desc(smem_u32(sm.kv[slot][0]), 16, 1024, kSwizzle128B);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_f16_ss(tmem + 16 * sb, kdesc + static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                       qdesc + static_cast<uint64_t>(((kk >> 2) * Smem::kRowBox + (kk & 3) * 32) >> 4), idS,
                       kk > 0 ? 1u : 0u);
          tc_commit(smem_u32(&sm.s_full[sb]));
          if (t + 1 == w.ntiles) tc_commit(smem_u32(&sm.q_empty[qb]));
          if (have_prev && !(ok = issue_pv())) break;
          have_prev = true;
          prev_slot = slot;
          prev_nu = nu;
          prev_t = t;
          prev_last = t + 1 == w.ntiles;
          ++kv_cons;
          ++g;
        }
        ++nu;
      }
      if (ok && have_prev) ok = issue_pv();
      if (!ok) sm.abort = 1;
      // every MMA issued so far must finish before TMEM is released
      tc_commit(smem_u32(&sm.drain));
      mbar_wait(smem_u32(&sm.drain), 0, nullptr, a.timeout_ns);
    }
  } else {
    // ======================= softmax warps 0-7 =======================
    const int grp = warp >> 2;  // group: takes the tiles with global index g, g % 2 == grp
    const int gtid = tid & 127;  // key of the tile = TMEM lane = output column in the epilogue
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_col = 16 * grp;
    const int bar_grp = kDecBarGroup + grp;
    const float cl = a.scale_log2;
    uint32_t g = 0, nu = 0;
    bool good = true;    // this warp's waits all succeeded (warp-uniform)
    bool failed = false;  // a barrier of this group saw a failure (group-uniform)
    auto wait = [&](uint64_t* bar, uint32_t parity, int site) {
      const bool w = __all_sync(0xffffffffu, mbar_wait(smem_u32(bar), parity, abort, a.timeout_ns));
      if (!w) {
        if (lane == 0) report_error(a.status, kStatusTimeout, site);
        sm.abort = 1;
      }
      good = good && w;
    };
    DecUnit w_next = dec_unit(a, blockIdx.x);
    for (int u = blockIdx.x; u < a.num_units; u += gridDim.x) {
      const DecUnit w = w_next;
      if (u + static_cast<int>(gridDim.x) < a.num_units) w_next = dec_unit(a, u + gridDim.x);
      if (w.ntiles == 0) {
        if (grp == 0) dec_write_empty<D>(a, w, gtid, G, R);
        continue;
      }
      // keys below lim_all are visible to every row; causal rows see fewer
      const int lim_all = a.causal ? min(w.k_end, w.Lb - a.Nq + 1) : w.k_end;
      float m[kDecRows], lp[kDecRows];
#pragma unroll
      for (int r = 0; r < kDecRows; ++r) {
        m[r] = -INFINITY;
        lp[r] = 0.f;
      }
      const uint32_t ob = nu & 1;
      const uint32_t o_col = 32 + 32 * grp + 16 * ob;
      int mine = 0;  // tiles of this unit taken by the group
      for (int t = 0; t < w.ntiles; ++t, ++g) {
        if ((g & 1) != static_cast<uint32_t>(grp) || failed) continue;
        wait(&sm.s_full[grp], (g >> 1) & 1, 97);
        float x[kDecRows];
        bool need = false;
        const int key = w.k_begin + t * kDecKeys + gtid;
        if (good) {
          tc_fence_after();
          uint32_t raw[16];
          tmem_ld16(tmem + lane_off + s_col, raw);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sm.s_free[grp]));
          if (w.k_begin + (t + 1) * kDecKeys <= lim_all) {
            // every key of the tile is visible to every row
#pragma unroll
            for (int r = 0; r < kDecRows; ++r) {
              x[r] = r < R ? __uint_as_float(raw[r]) * cl : -INFINITY;
              need |= x[r] > m[r] + kDecTau;
            }
          } else {
            // row r = i*G + g sees keys below min(k_end, L_b - Nq + i + 1)
            // when causal (i advanced by counting, no division)
            int i = 0, gg = 0;
#pragma unroll
            for (int r = 0; r < kDecRows; ++r) {
              const int lim = a.causal ? min(w.k_end, w.Lb - a.Nq + i + 1) : w.k_end;
              x[r] = (r < R && key < lim) ? __uint_as_float(raw[r]) * cl : -INFINITY;
              need |= x[r] > m[r] + kDecTau;
              if (++gg == G) {
                gg = 0;
                ++i;
              }
            }
          }
        }
        // The group's maximum is refreshed only when a score passes it by
        // more than the threshold (always on the group's first tile). The
        // group's previous tile (g-2) has finished its P V by now: the score
        // MMA of tile g was committed after that P V was issued, and a commit
        // completes only when everything issued before it has. So the P
        // buffer is free and the group's O^T may be rescaled.
        if (bar_red_or(need || !good, bar_grp, 128)) {
          if (good) {
            const float cm = warp_colreduce16<true>(x, lane);
            if ((lane & 1) == 0) sm.red_m[grp][lane >> 1][warp & 3] = cm;
          }
          if (!bar_red_and(good, bar_grp, 128)) {
            failed = true;  // skip the rest; the epilogue barrier ends both groups
            continue;
          }
          uint32_t o[16];
          if (mine > 0) {
            tc_fence_after();
            tmem_ld16(tmem + lane_off + o_col, o);
          }
#pragma unroll
          for (int r = 0; r < kDecRows; ++r) {
            const float4 c4 = *reinterpret_cast<const float4*>(sm.red_m[grp][r]);
            const float mn = fmaxf(m[r], fmaxf(fmaxf(c4.x, c4.y), fmaxf(c4.z, c4.w)));
            const float alpha = mn == -INFINITY ? 1.f : ex2_approx(m[r] - mn);
            lp[r] *= alpha;
            m[r] = mn;
            o[r] = __float_as_uint(__uint_as_float(o[r]) * alpha);
          }
          if (mine > 0) {
            tmem_st16(tmem + lane_off + o_col, o);
            tmem_st_wait();
          }
        }
        uint32_t pbits[kDecRows / 2];  // bf16 pairs: rows 2k (low half), 2k+1 (high half)
        if (good) {
#pragma unroll
          for (int r = 0; r < kDecRows; r += 2) {
            const float p0 = ex2_approx(x[r] - (m[r] == -INFINITY ? 0.f : m[r]));
            const float p1 = ex2_approx(x[r + 1] - (m[r + 1] == -INFINITY ? 0.f : m[r + 1]));
            lp[r] += p0;
            lp[r + 1] += p1;
            pbits[r / 2] = pack_bf16x2(p0, p1);
          }
        }
        if (good) {
          uint8_t* pbuf = &sm.p[grp][0][0];
#pragma unroll
          for (int r = 0; r < kDecRows; ++r)
            *reinterpret_cast<uint16_t*>(pbuf + dec_p_offset(r, gtid)) =
                static_cast<uint16_t>((r & 1) ? (pbits[r / 2] >> 16) : (pbits[r / 2] & 0xffffu));
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sm.p_full[grp]));
        }
        ++mine;
      }
      // ---- epilogue of the unit. Each group: row sums = column sums of the
      // per-key partials; then the groups swap (max, sums, tile counts).
      const int par = nu & 1;
      if (!failed && mine > 0) {
        if (good) {
          const float cs = warp_colreduce16<false>(lp, lane);
          if ((lane & 1) == 0) sm.red_l[grp][lane >> 1][warp & 3] = cs;
        }
        if (!bar_red_and(good, bar_grp, 128)) failed = true;
      }
      if (gtid == 0) {
#pragma unroll
        for (int r = 0; r < kDecRows; ++r) {
          const float4 c4 = *reinterpret_cast<const float4*>(sm.red_l[grp][r]);
          sm.xm[par][grp][r] = m[r];
          sm.xl[par][grp][r] = mine > 0 ? (c4.x + c4.y) + (c4.z + c4.w) : 0.f;
        }
        sm.xn[par][grp] = mine;
      }
      if (!bar_red_and(good && !failed, kDecBarSoftmax, 256)) break;
      const int n0 = sm.xn[par][0], n1 = sm.xn[par][1];
      wait(&sm.o_full[ob], (nu >> 1) & 1, 99);
      if (good) {
        // this group writes rows 8*grp .. 8*grp+7: columns 8*grp.. of both O^T
        tc_fence_after();
        uint32_t o0[8], o1[8];
        if (n0 > 0) tmem_ld8(tmem + lane_off + 32 + 16 * ob + 8 * grp, o0);
        if (n1 > 0) tmem_ld8(tmem + lane_off + 64 + 16 * ob + 8 * grp, o1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.o_empty[ob]));
        const size_t ps = static_cast<size_t>(w.split) * a.B * a.Nq * a.Hq;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int r = 8 * grp + c;
          if (r >= R) continue;
          const float m0 = sm.xm[par][0][r], m1 = sm.xm[par][1][r];
          const float mm = fmaxf(m0, m1);
          const float w0 = (n0 > 0 && m0 != -INFINITY) ? ex2_approx(m0 - mm) : 0.f;
          const float w1 = (n1 > 0 && m1 != -INFINITY) ? ex2_approx(m1 - mm) : 0.f;
          const float l = w0 * sm.xl[par][0][r] + w1 * sm.xl[par][1][r];
          float acc = 0.f;
          if (w0 != 0.f) acc = w0 * __uint_as_float(o0[c]);
          if (w1 != 0.f) acc = fmaf(w1, __uint_as_float(o1[c]), acc);
          const int i = r / G, hq = w.hk * G + (r - i * G);
          const size_t orow = (static_cast<size_t>(w.b) * a.Nq + i) * a.Hq + hq;
          const size_t li = (static_cast<size_t>(w.b) * a.Hq + hq) * a.Nq + i;
          const float val = l > 0.f ? acc / l : 0.f;
          const float lse = l > 0.f ? mm * 0.6931471805599453f + logf(l) : -INFINITY;
          if (a.splits == 1) {
            if (gtid < D) reinterpret_cast<__nv_bfloat16*>(a.o)[orow * D + gtid] = __float2bfloat16_rn(val);
            if (gtid == 0) a.lse[li] = lse;
          } else {
            if (gtid < D) a.part_o[(ps + orow) * D + gtid] = val;
            if (gtid == 0) a.part_lse[ps + li] = lse;
          }
        }
      }
      ++nu;
    }
  }

  // ---- teardown: every role is out of its loop; release TMEM
  tc_fence_before();
  __syncthreads();
  if (sm.abort && warp == kDecWarpProducer && lane == 0) {
    // after an abort, let the loads already issued land before the CTA exits
    for (uint32_t i = (prod_issued > ST ? prod_issued - ST : 0); i < prod_issued; ++i)
      mbar_wait(smem_u32(&sm.kv_full[i % ST]), (i / ST) & 1, nullptr, a.timeout_ns);
    for (uint32_t i = (q_issued > 2 ? q_issued - 2 : 0); i < q_issued; ++i)
      mbar_wait(smem_u32(&sm.q_full[i & 1]), (i >> 1) & 1, nullptr, a.timeout_ns);
  }
  __syncthreads();
  if (warp == kDecWarpMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// One warp per (batch, query, head) row. The lanes first stride over the
// splits for the maximum and the sum of exp(LSE_r - max); then each lane owns
// D/32 consecutive columns and accumulates the splits in order, several
// splits' loads in flight at once.
template <int D>
__global__ void __launch_bounds__(256) fa_decode_merge_kernel(const DecArgs a) {
  constexpr int PER = D / 32;
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(a.B) * a.Nq * a.Hq;
  const long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (w >= rows) return;
  const int hq = static_cast<int>(w % a.Hq);
  const int i = static_cast<int>((w / a.Hq) % a.Nq);
  const int b = static_cast<int>(w / (static_cast<long long>(a.Hq) * a.Nq));
  const size_t per_split = static_cast<size_t>(a.B) * a.Nq * a.Hq;
  const size_t li = (static_cast<size_t>(b) * a.Hq + hq) * a.Nq + i;
  const float* plse = a.part_lse + li;
  float m = -INFINITY;
  for (int r = lane; r < a.splits; r += 32) m = fmaxf(m, plse[r * per_split]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float lse = -INFINITY;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  if (m != -INFINITY) {
    float sum = 0.f;
    for (int r = lane; r < a.splits; r += 32) sum += expf(plse[r * per_split] - m);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    lse = m + logf(sum);
    const float* po = a.part_o + static_cast<size_t>(w) * D + lane * PER;
#pragma unroll 4
    for (int r = 0; r < a.splits; ++r) {
      const float wgt = expf(plse[r * per_split] - lse);  // 0 for an empty split
      const float* src = po + r * per_split * D;
      if constexpr (PER == 4) {
        const float4 v = *reinterpret_cast<const float4*>(src);
        acc[0] = fmaf(wgt, v.x, acc[0]);
        acc[1] = fmaf(wgt, v.y, acc[1]);
        acc[2] = fmaf(wgt, v.z, acc[2]);
        acc[3] = fmaf(wgt, v.w, acc[3]);
      } else {
        const float2 v = *reinterpret_cast<const float2*>(src);
        acc[0] = fmaf(wgt, v.x, acc[0]);
        acc[1] = fmaf(wgt, v.y, acc[1]);
      }
    }
  }
  __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.o) + static_cast<size_t>(w) * D + lane * PER;
  if constexpr (PER == 4)
    *reinterpret_cast<uint2*>(orow) = make_uint2(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]));
  else
    *reinterpret_cast<uint32_t*>(orow) = pack_bf16x2(acc[0], acc[1]);
  if (lane == 0) a.lse[li] = lse;
}

}  // namespace fa
