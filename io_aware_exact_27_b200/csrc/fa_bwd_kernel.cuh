// Backward pass of exact attention on sm_100a (bf16 in, fp32 accumulation),
// recomputing the scores from Q, K, V and the forward's LSE instead of storing
// P (catalogue record "Dao and colleagues: IO-aware exact attention with
// FlashAttention", summary: tiled operations and recomputation).
//
// Gradient of sum(O * dO), per (sequence, query head h, key/value head g):
//   P = exp(scale * Q K^T - LSE),  D_i = sum_c dO_ic O_ic,
//   dS = P * (dO V^T - D),  dV = P^T dO,  dK = scale * dS^T Q,  dQ = scale * dS K.
//
// Three kernels, deterministic by construction (no atomics, every output
// element is written once by one CTA):
//   fa_bwd_pre_kernel   D and LSE*log2(e) per query row into the workspace
//                       (fa_bwd_pre_kernel.cuh).
//   fa_bwd_dkdv_kernel  one CTA per (sequence, kv head, 128-key tile): walks
//                       the GQA group's query heads and query tiles, keeps
//                       S^T, dP^T, dV, dK in TMEM (4 x 128 columns).
//   fa_bwd_dq_kernel    one CTA per (sequence, query head, 128-row tile):
//                       recomputes S and dP per key block, dQ in TMEM.
// The dQ kernel recomputes S and dP (three GEMMs per tile pair instead of
// one), which keeps dQ free of cross-CTA reductions.
//
// Elementwise warps: 8 warps, two per TMEM lane quadrant; warp w handles the
// rows (lanes) 32*(w%4).. and the column half w/4 of each 128-column tile.
#pragma once

#include "fa_bwd_args.cuh"
#include "fa_tile.cuh"

namespace fa {

// Block-sparse backward (the forward's mask): key block kb visible to query
// block qb of query head hq. A dQ unit (query tile qt of head h) walks the key
// blocks it sees; a dK/dV unit (key tile kb of kv head hk) walks the (query
// head of the group, query tile) steps that see it, read from the step lists
// of the work plan (see fa_bwd_plan_kernel). A unit that sees none still runs
// one block / step, every score masked (zero gradient), so that every role
// runs the same pipeline.
__device__ __forceinline__ bool bwd_block_on(const BwdArgs& a, int hq, int qb, int kb) {
  return __ldg(a.block_mask + (static_cast<size_t>(hq) * a.nqb + qb) * a.nqb + kb) != 0;
}
// ------------------------------------------------------------------ dQ
template <int D, int STAGES, bool F8 = false>
struct DqSmem {
  static constexpr int kTileBytes = kBM * D * 2;
  static constexpr int kTile8 = kBM * D;  // a tile of e4m3 codes
  // bf16: Q; fp8: the Q codes (S = Q K^T on e4m3; Q itself is not needed)
  alignas(1024) uint8_t q[F8 ? kTile8 : kTileBytes];
  alignas(1024) uint8_t dout[kTileBytes];
  alignas(1024) uint8_t kv[STAGES][kTileBytes];
  // fp8: the K codes of the blocks whose bf16 K sits in kv[2 i]
  alignas(1024) uint8_t k8[F8 ? STAGES / 2 : 1][F8 ? kTile8 : 1024];
  uint64_t q_full, q_empty;
  uint64_t kv_full[STAGES], kv_empty[STAGES];
  uint64_t s_full[2], dp_full, ds_ready, acc_final, acc_free;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int level_count[1024];
};

// (split_a_col: the split TMEM A-operand layout, shared with the forward)

// D(M=128, N=DD) (+)= A(TMEM, 128 x 128 split halves) * B(smem [128 x DD] MN-major)
template <int DD>
__device__ __forceinline__ void issue_ts_split(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_smem, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBM, DD, false, true);
  const uint64_t bd = smem_desc(b_smem, 16384, 1024, kSwizzle128B);  // + (kk * 2048) >> 4 per step
  const uint32_t acc0 = accumulate ? 1u : 0u;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_f16_ts(d_tmem, a_tmem + split_a_col(kk), bd + static_cast<uint64_t>((kk * 2048) >> 4), idesc,
               kk > 0 ? 1u : acc0);
}

// D(128 x 128) = A(smem [128 x DD] K-major) * B(smem [128 x DD] K-major)^T
template <int DD>
__device__ __forceinline__ void issue_ss_nt(uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem) {
  issue_qk<DD>(d_tmem, a_smem, b_smem);
}

template <int D, int STAGES, bool SPARSE = false, bool F8 = false>
__global__ void __launch_bounds__(kThreadsBwd, 1)
    fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_q8, const __grid_constant__ CUtensorMap tm_k8,
                     const BwdArgs args) {
  static_assert(!(F8 && SPARSE), "fp8 backward is dense");
  using Smem = DqSmem<D, STAGES, F8>;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  if (tid == 0) {
    mbar_init(smem_u32(&sm.q_full), 1);
    mbar_init(smem_u32(&sm.q_empty), 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&sm.kv_full[s]), 1);
      mbar_init(smem_u32(&sm.kv_empty[s]), 1);
    }
    mbar_init(smem_u32(&sm.s_full[0]), 1);
    mbar_init(smem_u32(&sm.s_full[1]), 1);
    mbar_init(smem_u32(&sm.dp_full), 1);
    mbar_init(smem_u32(&sm.ds_ready), 8);
    mbar_init(smem_u32(&sm.acc_final), 1);
    mbar_init(smem_u32(&sm.acc_free), 8);
    mbar_init(smem_u32(&sm.drain), 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  const int nlevels = (args.N + 127) / 128;
  const bool varlen = args.cu_seqlens != nullptr;
  if (warp == 9) {
    tmem_alloc(smem_u32(&sm.tmem_base), 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tmap(F8 ? &tm_q8 : &tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_do);
    if constexpr (F8) prefetch_tmap(&tm_k8);
  }
  __syncthreads();
  int num_units = args.num_units;
  if (varlen)
    num_units = varlen_level_table(sm.level_count, args.cu_seqlens, args.nseq, nlevels, 7, args.Hq, kThreadsBwd);
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  // TMEM: S0 [0,128) S1 [128,256) dP [256,384) dQ [384, 384+D)
  const uint32_t tS0 = tmem, tDP = tmem + 256, tDQ = tmem + 384;
  SeqSched sched{args.cu_seqlens, args.nseq, args.N, args.Hq, !args.causal, nlevels, sm.level_count, 7,
                 !SPARSE && !varlen && !args.causal};
  const volatile int* abort = &sm.abort;
  const int group = args.Hq / args.Hkv;
  uint32_t prod_issued = 0, q_issued = 0;
  // block-sparse: the unit's row of key blocks (count, first list entry);
  // a row that sees nothing still visits block 0, every score masked
  auto row_of = [&](const Unit& un, int& rn, int& rb) {
    rn = 0;
    rb = 0;
    if constexpr (SPARSE) {
      const int r = un.h * args.nqb + un.qb2;
      rn = __ldg(args.rows_n + r);
      rb = __ldg(args.rows_base + r);
    }
  };
  auto block_at = [&](int rn, int rb, int j) -> int {
    if constexpr (SPARSE)
      return rn > 0 ? __ldg(args.rows_list + rb + j) : 0;
    else
      return j;
  };

  if (warp == 8) {
    if (lane == 0) {
      uint32_t kv_prod = 0, it = 0;
      bool ok = true;
      for (int rnd = 0; ok; ++rnd, ++it) {
        const int u = unit_of(rnd, blockIdx.x, gridDim.x);
        if (u >= num_units) break;
        const Unit un = decode_unit(sched, u);
        const int jend = args.causal ? min((un.n + 127) / 128, un.qb2 + 1) : (un.n + 127) / 128;
        int rn, rb;
        row_of(un, rn, rb);
        const int nblk = SPARSE ? max(rn, 1) : jend;  // blocks visited
        const int hkv = un.h / group;
        if (!mbar_wait(smem_u32(&sm.q_empty), (it & 1) ^ 1, abort, args.timeout_ns)) {
          report_error(args.status, kStatusTimeout, 30);
          ok = false;
          break;
        }
        const uint32_t qbar = smem_u32(&sm.q_full);
        mbar_expect_tx(qbar, (F8 ? Smem::kTile8 : Smem::kTileBytes) + Smem::kTileBytes);
        const int row0 = un.tok0 + un.qb2 * kBM;
        if constexpr (F8)
          load_tile<D, 1>(smem_u32(sm.q), &tm_q8, qbar, un.h, row0);
        else
          load_tile<D>(smem_u32(sm.q), &tm_q, qbar, un.h, row0);
        load_tile<D>(smem_u32(sm.dout), &tm_do, qbar, un.h, row0);
        q_issued = it + 1;
        for (int j = 0; j < nblk && ok; ++j) {
          const int jb = block_at(rn, rb, j);  // key block of the j-th visit
          for (int kv = 0; kv < 2; ++kv) {
            const uint32_t slot = kv_prod % STAGES;
            if (!mbar_wait(smem_u32(&sm.kv_empty[slot]), ((kv_prod / STAGES) & 1) ^ 1, abort, args.timeout_ns)) {
              report_error(args.status, kStatusTimeout, 31);
              ok = false;
              break;
            }
            const uint32_t bar = smem_u32(&sm.kv_full[slot]);
            // fp8: a K slot also receives the block's K codes (K slots are the even ones)
            mbar_expect_tx(bar, Smem::kTileBytes + (F8 && kv == 0 ? Smem::kTile8 : 0));
            load_tile<D>(smem_u32(sm.kv[slot]), kv == 0 ? &tm_k : &tm_v, bar, hkv, un.tok0 + jb * kBN);
            if constexpr (F8)
              if (kv == 0) load_tile<D, 1>(smem_u32(sm.k8[slot / 2]), &tm_k8, bar, hkv, un.tok0 + jb * kBN);
            ++kv_prod;
          }
        }
      }
      if (!ok) sm.abort = 1;
      prod_issued = kv_prod;
    }
  } else if (warp == 9) {
    if (lane == 0) {
      uint32_t kv_cons = 0, it = 0, dsc = 0, sb_cnt = 0;
      bool ok = true;
      auto wait = [&](uint64_t* bar, uint32_t parity, int site) -> bool {
        if (!mbar_wait(smem_u32(bar), parity, abort, args.timeout_ns)) {
          report_error(args.status, kStatusTimeout, site);
          return false;
        }
        tc_fence_after();
        return true;
      };
      (void)sb_cnt;
      for (int rnd = 0; ok; ++rnd, ++it) {
        const int u = unit_of(rnd, blockIdx.x, gridDim.x);
        if (u >= num_units) break;
        const Unit un = decode_unit(sched, u);
        const int jend = args.causal ? min((un.n + 127) / 128, un.qb2 + 1) : (un.n + 127) / 128;
        int rn, rb;
        row_of(un, rn, rb);
        const int nblk = SPARSE ? max(rn, 1) : jend;  // blocks visited
        (void)rb;
        if (!(ok = wait(&sm.q_full, it & 1, 40))) break;
        const uint32_t qa = smem_u32(sm.q), doa = smem_u32(sm.dout);
        // prologue: S(0)
        uint32_t slotK = kv_cons % STAGES;
        if (!(ok = wait(&sm.kv_full[slotK], (kv_cons / STAGES) & 1, 41))) break;
        ++kv_cons;
        auto issue_s = [&](uint32_t d_tmem, uint32_t slot) {
          if constexpr (F8)
            issue_qk<D, true>(d_tmem, qa, smem_u32(sm.k8[slot / 2]));  // e4m3 codes
          else
            issue_ss_nt<D>(d_tmem, qa, smem_u32(sm.kv[slot]));
        };
        issue_s(tS0, slotK);
        tc_commit(smem_u32(&sm.s_full[0]));
        for (int j = 0; j < nblk; ++j) {
          const uint32_t slotV = kv_cons % STAGES;
          if (!(ok = wait(&sm.kv_full[slotV], (kv_cons / STAGES) & 1, 42))) break;
          ++kv_cons;
          // dP(j) = dO V_j^T
          issue_ss_nt<D>(tDP, doa, smem_u32(sm.kv[slotV]));
          tc_commit(smem_u32(&sm.dp_full));
          tc_commit(smem_u32(&sm.kv_empty[slotV]));
          uint32_t slotKn = 0;
          if (j + 1 < nblk) {
            slotKn = kv_cons % STAGES;
            if (!(ok = wait(&sm.kv_full[slotKn], (kv_cons / STAGES) & 1, 43))) break;
            ++kv_cons;
            issue_s(tS0 + ((j + 1) & 1) * 128, slotKn);
            tc_commit(smem_u32(&sm.s_full[(j + 1) & 1]));
          }
          if (j + 1 == nblk) tc_commit(smem_u32(&sm.q_empty));  // last reads of Q and dO issued
          // dQ += dS K_j
          if (!(ok = wait(&sm.ds_ready, dsc & 1, 44))) break;
          ++dsc;
          if (j == 0 && !(ok = wait(&sm.acc_free, (it & 1) ^ 1, 45))) break;
          issue_ts_split<D>(tDQ, tDP, smem_u32(sm.kv[slotK]), j > 0);
          tc_commit(smem_u32(&sm.kv_empty[slotK]));
          slotK = slotKn;
        }
        if (!ok) break;
        tc_commit(smem_u32(&sm.acc_final));
      }
      if (!ok) sm.abort = 1;
      tc_commit(smem_u32(&sm.drain));
      mbar_wait(smem_u32(&sm.drain), 0, nullptr, args.timeout_ns);
    }
  } else {
    // ---------------- elementwise warps
    const int half = warp >> 2;
    const int quad = warp & 3;
    const int r_in_tile = quad * 32 + lane;
    const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
    const float cl = args.scale_log2;
    uint32_t sc0 = 0, sc1 = 0, dpc = 0, it = 0;
    bool ok = true;
    for (int rnd = 0; ok; ++rnd, ++it) {
      const int u = unit_of(rnd, blockIdx.x, gridDim.x);
      if (u >= num_units) break;
      const Unit un = decode_unit(sched, u);
      const int jend = args.causal ? min((un.n + 127) / 128, un.qb2 + 1) : (un.n + 127) / 128;
      int rn, rb;
      row_of(un, rn, rb);
      const int nblk = SPARSE ? max(rn, 1) : jend;  // blocks visited
      const int row = un.qb2 * kBM + r_in_tile;
      const bool valid = row < un.n;
      const size_t wi = static_cast<size_t>(un.h) * args.ws_stride + ws_offset(un.tok0, un.seq) + row;
      const float lse2 = valid ? args.lse2[wi] : INFINITY;
      const float dval = valid ? args.dvec[wi] : 0.f;
      const int limit = args.causal ? min(row, un.n - 1) : un.n - 1;
      // fp8: the scores are in code units, scaled by the Q and K block scales
      const float* kscale = nullptr;
      float cq = cl;
      if constexpr (F8) {
        cq = cl * args.q_scale[(static_cast<size_t>(un.seq) * args.Hq + un.h) * args.nblk_s + un.qb2];
        kscale = args.k_scale + (static_cast<size_t>(un.seq) * args.Hkv + un.h / group) * args.nblk_s;
      }
      for (int j = 0; j < nblk; ++j) {
        const int jb = block_at(rn, rb, j);  // key block of the j-th visit
        const int sb = j & 1;
        const float cj = F8 ? cq * kscale[jb] : cl;
        const uint32_t par = sb ? (sc1 & 1) : (sc0 & 1);
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.s_full[sb]), par, abort, args.timeout_ns));
        if (!ok) {
          if (lane == 0) report_error(args.status, kStatusTimeout, 50);
          break;
        }
        if (sb) ++sc1; else ++sc0;
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld64(tS0 + sb * 128 + half * 64 + lane_bits, sr);
        float p[64];
        const int c0 = jb * kBN + half * 64;
        // block-sparse: a visit of a block this tile may not see (a unit that sees none)
        const bool off = SPARSE && rn == 0;
        const bool masked_blk = off || __any_sync(0xffffffffu, c0 + 63 > limit);
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float x = ex2_approx(fmaf(__uint_as_float(sr[c]), cj, -lse2));
          p[c] = (masked_blk && (off || c0 + c > limit)) ? 0.f : x;
        }
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.dp_full), dpc & 1, abort, args.timeout_ns));
        if (!ok) {
          if (lane == 0) report_error(args.status, kStatusTimeout, 51);
          break;
        }
        ++dpc;
        tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t dr[32];
          tmem_ld32(tDP + half * 64 + ch * 32 + lane_bits, dr);
          uint32_t pk[16];
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const float a0 = p[ch * 32 + 2 * t] * (__uint_as_float(dr[2 * t]) - dval);
            const float a1 = p[ch * 32 + 2 * t + 1] * (__uint_as_float(dr[2 * t + 1]) - dval);
            pk[t] = pack_bf16x2(a0, a1);
          }
          tmem_st16(tDP + half * 64 + ch * 16 + lane_bits, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.ds_ready));
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.acc_final), it & 1, abort, args.timeout_ns));
      if (!ok) {
        if (lane == 0) report_error(args.status, kStatusTimeout, 52);
        break;
      }
      tc_fence_after();
      constexpr int HC = D / 2;  // dQ columns per half
      __nv_bfloat16* qrow = reinterpret_cast<__nv_bfloat16*>(args.dq) +
                            (static_cast<size_t>(un.tok0 + row) * args.Hq + un.h) * D + half * HC;
#pragma unroll
      for (int c = 0; c < HC; c += 32) {
        uint32_t orr[32];
        tmem_ld32(tDQ + half * HC + c + lane_bits, orr);
        uint32_t pk[16];
#pragma unroll
        for (int t = 0; t < 16; ++t)
          pk[t] = pack_bf16x2(__uint_as_float(orr[2 * t]) * args.scale, __uint_as_float(orr[2 * t + 1]) * args.scale);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(qrow + c);
#pragma unroll
          for (int t = 0; t < 4; ++t) dst[t] = make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.acc_free));
    }
    if (!ok) sm.abort = 1;
  }

  tc_fence_before();
  __syncthreads();
  if (sm.abort && warp == 8 && lane == 0) {
    for (uint32_t i = (prod_issued > STAGES ? prod_issued - STAGES : 0); i < prod_issued; ++i)
      mbar_wait(smem_u32(&sm.kv_full[i % STAGES]), (i / STAGES) & 1, nullptr, args.timeout_ns);
    if (q_issued > 0) mbar_wait(smem_u32(&sm.q_full), (q_issued - 1) & 1, nullptr, args.timeout_ns);
  }
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ dK, dV
template <int D, int STAGES, bool F8 = false>
struct DkvSmem {
  static constexpr int kTileBytes = kBM * D * 2;
  static constexpr int kTile8 = kBM * D;  // a tile of e4m3 codes
  alignas(1024) uint8_t k[F8 ? kTile8 : kTileBytes];  // K (fp8: its codes, for S^T only)
  alignas(1024) uint8_t v[kTileBytes];
  alignas(1024) uint8_t qo[STAGES][kTileBytes];  // Q_i, dO_i alternating
  // fp8: the step's Q codes (S^T = K Q^T on e4m3), one per step of the ring
  alignas(1024) uint8_t q8[F8 ? STAGES / 2 : 1][F8 ? kTile8 : 1024];
  alignas(16) float vec[STAGES / 2][2][128];     // per step: LSE2, D of the 128 query columns
  uint64_t kv_full, kv_empty;
  uint64_t qo_full[STAGES], qo_empty[STAGES];
  uint64_t s_full, dp_full, p_ready, ds_ready, acc_final, acc_free;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int level_count[1024];
};

template <int D, int STAGES, bool SPARSE = false, bool F8 = false>
__global__ void __launch_bounds__(kThreadsBwd, 1)
    fa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_q8, const __grid_constant__ CUtensorMap tm_k8,
                       const BwdArgs args) {
  static_assert(STAGES % 2 == 0, "Q and dO alternate in the ring");
  static_assert(!(F8 && SPARSE), "fp8 backward is dense");
  using Smem = DkvSmem<D, STAGES, F8>;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  if (tid == 0) {
    mbar_init(smem_u32(&sm.kv_full), 1);
    mbar_init(smem_u32(&sm.kv_empty), 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&sm.qo_full[s]), 1);
      mbar_init(smem_u32(&sm.qo_empty[s]), 1);
    }
    mbar_init(smem_u32(&sm.s_full), 1);
    mbar_init(smem_u32(&sm.dp_full), 1);
    mbar_init(smem_u32(&sm.p_ready), 8);
    mbar_init(smem_u32(&sm.ds_ready), 8);
    mbar_init(smem_u32(&sm.acc_final), 1);
    mbar_init(smem_u32(&sm.acc_free), 8);
    mbar_init(smem_u32(&sm.drain), 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  const int nlevels = (args.N + 127) / 128;
  const bool varlen = args.cu_seqlens != nullptr;
  if (warp == 9) {
    tmem_alloc(smem_u32(&sm.tmem_base), 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(F8 ? &tm_k8 : &tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_do);
    if constexpr (F8) prefetch_tmap(&tm_q8);
  }
  __syncthreads();
  int num_units = args.num_units;
  if (varlen)
    num_units = varlen_level_table(sm.level_count, args.cu_seqlens, args.nseq, nlevels, 7, args.Hkv, kThreadsBwd);
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  // TMEM: S^T [0,128) dP^T [128,256) dV [256,256+D) dK [384,384+D)
  const uint32_t tS = tmem, tDP = tmem + 128, tDV = tmem + 256, tDK = tmem + 384;
  // causal: the heaviest key tiles are the first ones (most query tiles see them)
  SeqSched sched{args.cu_seqlens, args.nseq, args.N, args.Hkv, args.causal, nlevels, sm.level_count, 7,
                 !SPARSE && !varlen && !args.causal};
  const volatile int* abort = &sm.abort;
  const int group = args.Hq / args.Hkv;
  uint32_t prod_issued = 0, kv_issued = 0;

  // steps of a unit: (query head of the group, query tile) pairs
  // (block-sparse: only the steps whose (query tile, key tile) block is on
  // are visited, at least one per unit so that dK and dV are written)
  auto unit_steps = [&](const Unit& un, int& i0, int& nqt) {
    const int nq = (un.n + 127) / 128;
    i0 = args.causal ? un.qb2 : 0;
    nqt = nq - i0;
    return group * nqt;
  };
  // work item w: block-sparse, the planned (unit, position of its first step
  // in the planned step list or -1 for a key tile nothing sees, steps,
  // partial slot or -1); dense, unit w whole
  const int nwork = SPARSE ? __ldg(args.plan) : num_units;
  auto work_of = [&](int w) -> int4 {
    if constexpr (SPARSE)
      return __ldg(reinterpret_cast<const int4*>(args.plan) + 1 + w);
    else
      return make_int4(w, 0, 0, -1);
  };
  // step v of an item
  auto step_of = [&](const int4& wk, int v) -> int {
    if constexpr (SPARSE)
      return wk.y < 0 ? 0 : __ldg(args.plan_steps + wk.y + v);
    else
      return v;
  };

  if (warp == 8) {
    uint32_t qo_prod = 0, it = 0;
    bool ok = true;
    for (int rnd = 0; ok; ++rnd, ++it) {
      const int w = unit_of(rnd, blockIdx.x, gridDim.x);
      if (w >= nwork) break;
      const int4 wk = work_of(w);
      const Unit un = decode_unit(sched, wk.x);
      int i0, nqt;
      const int nsteps = unit_steps(un, i0, nqt);
      const int nvis = SPARSE ? wk.z : nsteps;
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.kv_empty), (it & 1) ^ 1, abort, args.timeout_ns));
      if (!ok) {
        if (lane == 0) report_error(args.status, kStatusTimeout, 60);
        break;
      }
      if (lane == 0) {
        const uint32_t bar = smem_u32(&sm.kv_full);
        mbar_expect_tx(bar, (F8 ? Smem::kTile8 : Smem::kTileBytes) + Smem::kTileBytes);
        if constexpr (F8)
          load_tile<D, 1>(smem_u32(sm.k), &tm_k8, bar, un.h, un.tok0 + un.qb2 * kBN);
        else
          load_tile<D>(smem_u32(sm.k), &tm_k, bar, un.h, un.tok0 + un.qb2 * kBN);
        load_tile<D>(smem_u32(sm.v), &tm_v, bar, un.h, un.tok0 + un.qb2 * kBN);
      }
      kv_issued = it + 1;
      for (int v = 0; v < nvis && ok; ++v) {
        const int st = step_of(wk, v);
        const int hq = un.h * group + st / nqt;
        const int qi = i0 + st % nqt;
        for (int w = 0; w < 2; ++w) {
          const uint32_t slot = qo_prod % STAGES;
          ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.qo_empty[slot]), ((qo_prod / STAGES) & 1) ^ 1, abort,
                                                 args.timeout_ns));
          if (!ok) {
            if (lane == 0) report_error(args.status, kStatusTimeout, 61);
            break;
          }
          if (lane == 0) {
            // a step's Q and dO tiles and the query tile's LSE2 and D all
            // complete on the Q slot's barrier (Q sits in the even ring
            // slots): one wait covers the step for the MMA issuer, where
            // every mbarrier wait costs tensor-pipe time
            const uint32_t bar = smem_u32(&sm.qo_full[w == 0 ? slot : (slot + STAGES - 1) % STAGES]);
            if (w == 0) {
              float* vec = sm.vec[(qo_prod / 2) % (STAGES / 2)][0];
              const size_t wbase = static_cast<size_t>(hq) * args.ws_stride + ws_offset(un.tok0, un.seq) + qi * kBM;
              mbar_expect_tx(bar, 2 * Smem::kTileBytes + 1024 + (F8 ? Smem::kTile8 : 0));
              bulk_load(smem_u32(vec), args.lse2 + wbase, 512, bar);
              bulk_load(smem_u32(vec + 128), args.dvec + wbase, 512, bar);
              if constexpr (F8)
                load_tile<D, 1>(smem_u32(sm.q8[(qo_prod / 2) % (STAGES / 2)]), &tm_q8, bar, hq, un.tok0 + qi * kBM);
            }
            load_tile<D>(smem_u32(sm.qo[slot]), w == 0 ? &tm_q : &tm_do, bar, hq, un.tok0 + qi * kBM);
          }
          ++qo_prod;
        }
      }
    }
    if (!ok && lane == 0) sm.abort = 1;
    prod_issued = qo_prod;
  } else if (warp == 9) {
    if (lane == 0) {
      uint32_t qo_cons = 0, it = 0, pc = 0, dsc = 0;
      bool ok = true;
      auto wait = [&](uint64_t* bar, uint32_t parity, int site) -> bool {
        if (!mbar_wait(smem_u32(bar), parity, abort, args.timeout_ns)) {
          report_error(args.status, kStatusTimeout, site);
          return false;
        }
        tc_fence_after();
        return true;
      };
      for (int rnd = 0; ok; ++rnd, ++it) {
        const int w = unit_of(rnd, blockIdx.x, gridDim.x);
        if (w >= nwork) break;
        const int4 wk = work_of(w);
        const Unit un = decode_unit(sched, wk.x);
        int i0, nqt;
        const int nall = unit_steps(un, i0, nqt);
        const int nsteps = SPARSE ? wk.z : nall;  // visited
        if (!(ok = wait(&sm.kv_full, it & 1, 70))) break;
        const uint32_t ka = smem_u32(sm.k), va = smem_u32(sm.v);
        // prologue: S^T(0), dP^T(0)
        uint32_t slotQ = qo_cons % STAGES;
        if (!(ok = wait(&sm.qo_full[slotQ], (qo_cons / STAGES) & 1, 71))) break;
        uint32_t slotO = (qo_cons + 1) % STAGES;
        // S^T = K Q^T (fp8: on the codes; the step's Q codes sit in q8[slot / 2])
        auto issue_st = [&](uint32_t slot) {
          if constexpr (F8)
            issue_qk<D, true>(tS, ka, smem_u32(sm.q8[slot / 2]));
          else
            issue_ss_nt<D>(tS, ka, smem_u32(sm.qo[slot]));
        };
        issue_st(slotQ);
        tc_commit(smem_u32(&sm.s_full));
        issue_ss_nt<D>(tDP, va, smem_u32(sm.qo[slotO]));
        tc_commit(smem_u32(&sm.dp_full));
        if (nsteps == 1) tc_commit(smem_u32(&sm.kv_empty));  // last reads of K and V issued
        qo_cons += 2;
        for (int st = 0; st < nsteps; ++st) {
          const bool has_next = st + 1 < nsteps;
          // dV += P^T dO
          if (!(ok = wait(&sm.p_ready, pc & 1, 73))) break;
          ++pc;
          if (st == 0 && !(ok = wait(&sm.acc_free, (it & 1) ^ 1, 74))) break;
          issue_ts_split<D>(tDV, tS, smem_u32(sm.qo[slotO]), st > 0);
          tc_commit(smem_u32(&sm.qo_empty[slotO]));  // dO_st: last use
          uint32_t nQ = 0, nO = 0;
          if (has_next) {
            nQ = qo_cons % STAGES;
            nO = (qo_cons + 1) % STAGES;
            if (!(ok = wait(&sm.qo_full[nQ], (qo_cons / STAGES) & 1, 75))) break;
            issue_st(nQ);
            tc_commit(smem_u32(&sm.s_full));
          }
          // dK += dS^T Q
          if (!(ok = wait(&sm.ds_ready, dsc & 1, 76))) break;
          ++dsc;
          issue_ts_split<D>(tDK, tDP, smem_u32(sm.qo[slotQ]), st > 0);
          tc_commit(smem_u32(&sm.qo_empty[slotQ]));  // Q_st: last use
          if (has_next) {
            issue_ss_nt<D>(tDP, va, smem_u32(sm.qo[nO]));
            tc_commit(smem_u32(&sm.dp_full));
            // K and V are last read by this unit's final S^T and dP^T: release
            // them now so the next unit's tiles load under the last steps
            if (st + 2 == nsteps) tc_commit(smem_u32(&sm.kv_empty));
            qo_cons += 2;
            slotQ = nQ;
            slotO = nO;
          }
        }
        if (!ok) break;
        tc_commit(smem_u32(&sm.acc_final));
      }
      if (!ok) sm.abort = 1;
      tc_commit(smem_u32(&sm.drain));
      mbar_wait(smem_u32(&sm.drain), 0, nullptr, args.timeout_ns);
    }
  } else {
    // ---------------- elementwise warps: thread = key row, half = query column half
    const int half = warp >> 2;
    const int quad = warp & 3;
    const int r_in_tile = quad * 32 + lane;
    const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
    const float cl = args.scale_log2;
    uint32_t sc = 0, dpc = 0, it = 0, vstep = 0;
    bool ok = true;
    for (int rnd = 0; ok; ++rnd, ++it) {
      const int w = unit_of(rnd, blockIdx.x, gridDim.x);
      if (w >= nwork) break;
      const int4 wk = work_of(w);
      const Unit un = decode_unit(sched, wk.x);
      int i0, nqt;
      const int nsteps = unit_steps(un, i0, nqt);
      const int nvis = SPARSE ? wk.z : nsteps;
      const int key = un.qb2 * kBN + r_in_tile;  // key row within the sequence
      const bool valid = key < un.n;
      for (int v = 0; v < nvis; ++v, ++vstep) {
        const int st = step_of(wk, v);
        const int qi = i0 + st % nqt;
        // fp8: the scores are in code units, scaled by the Q and K block scales
        float cs = cl;
        if constexpr (F8)
          cs = cl * args.q_scale[(static_cast<size_t>(un.seq) * args.Hq + un.h * group + st / nqt) * args.nblk_s + qi] *
               args.k_scale[(static_cast<size_t>(un.seq) * args.Hkv + un.h) * args.nblk_s + un.qb2];
        // block-sparse: the forced visit of a key tile that no query tile sees
        const bool off = SPARSE && wk.y < 0;
        const float* vec = sm.vec[vstep % (STAGES / 2)][0];
        const int q0 = qi * kBM + half * 64;  // first query column of this half
        // the producer stored this step's LSE2/D before arriving on the Q
        // tile's barrier: waiting on it makes those stores visible here
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.qo_full[(2 * vstep) % STAGES]),
                                               ((2 * vstep) / STAGES) & 1, abort, args.timeout_ns));
        if (!ok) {
          if (lane == 0) report_error(args.status, kStatusTimeout, 83);
          break;
        }
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.s_full), sc & 1, abort, args.timeout_ns));
        if (!ok) {
          if (lane == 0) report_error(args.status, kStatusTimeout, 80);
          break;
        }
        ++sc;
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld64(tS + half * 64 + lane_bits, sr);
        // a query column q is hidden from key k when q >= n or (causal and k > q)
        const int lo = args.causal ? key : 0;  // smallest visible query
        const bool masked_blk = off || __any_sync(0xffffffffu, q0 < lo || q0 + 63 >= un.n);
        float p[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float x = ex2_approx(fmaf(__uint_as_float(sr[c]), cs, -vec[half * 64 + c]));
          p[c] = (masked_blk && (off || q0 + c < lo || q0 + c >= un.n)) ? 0.f : x;
        }
        {
          uint32_t pk[32];
#pragma unroll
          for (int t = 0; t < 32; ++t) pk[t] = pack_bf16x2(p[2 * t], p[2 * t + 1]);
          tmem_st32(tS + half * 64 + lane_bits, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.p_ready));
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.dp_full), dpc & 1, abort, args.timeout_ns));
        if (!ok) {
          if (lane == 0) report_error(args.status, kStatusTimeout, 81);
          break;
        }
        ++dpc;
        tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t dr[32];
          tmem_ld32(tDP + half * 64 + ch * 32 + lane_bits, dr);
          uint32_t pk[16];
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const int c = ch * 32 + 2 * t;
            const float a0 = p[c] * (__uint_as_float(dr[2 * t]) - vec[128 + half * 64 + c]);
            const float a1 = p[c + 1] * (__uint_as_float(dr[2 * t + 1]) - vec[128 + half * 64 + c + 1]);
            pk[t] = pack_bf16x2(a0, a1);
          }
          tmem_st16(tDP + half * 64 + ch * 16 + lane_bits, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.ds_ready));
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.acc_final), it & 1, abort, args.timeout_ns));
      if (!ok) {
        if (lane == 0) report_error(args.status, kStatusTimeout, 82);
        break;
      }
      tc_fence_after();
      constexpr int HC = D / 2;
      const size_t rowoff = (static_cast<size_t>(un.tok0 + key) * args.Hkv + un.h) * D + half * HC;
      for (int which = 0; which < 2; ++which) {
        __nv_bfloat16* dst_row = reinterpret_cast<__nv_bfloat16*>(which == 0 ? args.dv : args.dk) + rowoff;
        const uint32_t src = (which == 0 ? tDV : tDK) + half * HC + lane_bits;
        const float mul = which == 0 ? 1.f : args.scale;
#pragma unroll
        for (int c = 0; c < HC; c += 32) {
          uint32_t orr[32];
          tmem_ld32(src + c, orr);
          if (SPARSE && wk.w >= 0) {
            // a chunk of a split unit: its fp32 sums to its partial slot
            float4* prow = reinterpret_cast<float4*>(args.partials +
                                                     ((static_cast<size_t>(wk.w) * 2 + which) * kBN + r_in_tile) * D +
                                                     half * HC + c);
#pragma unroll
            for (int t = 0; t < 8; ++t)
              prow[t] = make_float4(__uint_as_float(orr[4 * t]), __uint_as_float(orr[4 * t + 1]),
                                    __uint_as_float(orr[4 * t + 2]), __uint_as_float(orr[4 * t + 3]));
            continue;
          }
          uint32_t pk[16];
#pragma unroll
          for (int t = 0; t < 16; ++t)
            pk[t] = pack_bf16x2(__uint_as_float(orr[2 * t]) * mul, __uint_as_float(orr[2 * t + 1]) * mul);
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(dst_row + c);
#pragma unroll
            for (int t = 0; t < 4; ++t) dst[t] = make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.acc_free));
    }
    if (!ok) sm.abort = 1;
  }

  tc_fence_before();
  __syncthreads();
  if (sm.abort && warp == 8 && lane == 0) {
    // (only the Q slots' barriers complete: a step's dO load counts on its Q slot)
    for (uint32_t i = (prod_issued > STAGES ? prod_issued - STAGES : 0); i < prod_issued; ++i)
      if ((i & 1) == 0) mbar_wait(smem_u32(&sm.qo_full[i % STAGES]), (i / STAGES) & 1, nullptr, args.timeout_ns);
    if (kv_issued > 0) mbar_wait(smem_u32(&sm.kv_full), (kv_issued - 1) & 1, nullptr, args.timeout_ns);
  }
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ block-sparse dK/dV plan
// With a block mask the dK/dV units can be very uneven (a key block every
// query block sees, e.g. a global first block, makes a unit group x nqb steps
// long against a handful for the others), and the CTA that holds such a unit
// bounds the kernel. fa_bwd_plan_count_kernel counts every unit's visible
// steps n_u; one CTA then takes
// a chunk length L = max(16, min(ceil(sum n / grid), ceil(sum n / units)))
// (the average unit, or the per-CTA share when there are fewer units than
// CTAs); a unit with n_u > 2L becomes ceil(n_u / L) chunks of (nearly) equal
// step counts, so that the items dealt round-robin to the CTAs are of about
// equal size. A split unit's chunks write fp32 partial dK/dV into their own
// slots, which fa_bwd_reduce_kernel sums in chunk order (deterministic). The
// slots are bounded (max_slots): a run of units whose chunks would not fit
// stays unsplit. A dense or causal mask never splits (no unit is twice the
// average).
constexpr int kPlanThreads = 1024;
constexpr int kPlanMinChunk = 16;
// Visible steps of every dK/dV unit (at least 1, the forced visit of a unit
// nothing sees), one warp per unit: the lanes test 32 steps at a time.
__global__ void __launch_bounds__(256) fa_bwd_plan_count_kernel(const BwdArgs a, int units, int* nbuf) {
  const int u = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (u >= units) return;  // uniform over the warp
  const int group = a.Hq / a.Hkv;
  const int nlevels = (a.N + 127) / 128;
  const SeqSched sched{nullptr, a.nseq, a.N, a.Hkv, a.causal, nlevels, nullptr, 7};
  const Unit un = decode_unit(sched, u);
  const int i0 = a.causal ? un.qb2 : 0;
  const int nqt = (un.n + 127) / 128 - i0;
  int n = 0;
  for (int base = 0; base < group * nqt; base += 32) {
    const int st = base + lane;
    const bool on = st < group * nqt && bwd_block_on(a, un.h * group + st / nqt, i0 + st % nqt, un.qb2);
    n += __popc(__ballot_sync(0xffffffffu, on));
  }
  if (lane == 0) nbuf[u] = n;
}

// Writes the visible steps of unit u at plan_steps[plan_sbase[u] ...], in
// step order (one warp per unit: ballot, then each set lane's rank).
__global__ void __launch_bounds__(256) fa_bwd_plan_steps_kernel(const BwdArgs a, int units) {
  const int u = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (u >= units) return;  // uniform over the warp
  const int group = a.Hq / a.Hkv;
  const int nlevels = (a.N + 127) / 128;
  const SeqSched sched{nullptr, a.nseq, a.N, a.Hkv, a.causal, nlevels, nullptr, 7};
  const Unit un = decode_unit(sched, u);
  const int i0 = a.causal ? un.qb2 : 0;
  const int nqt = (un.n + 127) / 128 - i0;
  int pos = a.plan_sbase[u];
  for (int base = 0; base < group * nqt; base += 32) {
    const int st = base + lane;
    const bool on = st < group * nqt && bwd_block_on(a, un.h * group + st / nqt, i0 + st % nqt, un.qb2);
    const uint32_t bal = __ballot_sync(0xffffffffu, on);
    if (on) a.plan_steps[pos + __popc(bal & ((1u << lane) - 1u))] = st;
    pos += __popc(bal);
  }
}

__global__ void __launch_bounds__(kPlanThreads) fa_bwd_plan_kernel(const BwdArgs a, int units, int grid, int max_slots,
                                                                   const int* nbuf) {
  __shared__ long long red[kPlanThreads];
  __shared__ int scan_items[kPlanThreads], scan_slots[kPlanThreads], scan_splits[kPlanThreads];
  __shared__ int scan_steps[kPlanThreads];
  __shared__ unsigned char nosplit[kPlanThreads];
  const int tid = threadIdx.x;
  long long local = 0;
  for (int u = tid; u < units; u += kPlanThreads) local += nbuf[u];
  red[tid] = local;
  __syncthreads();
  for (int off = kPlanThreads / 2; off > 0; off >>= 1) {
    if (tid < off) red[tid] += red[tid + off];
    __syncthreads();
  }
  const long long total = red[0];
  const long long share = (total + grid - 1) / grid, avg = (total + units - 1) / units;
  const long long L = max(static_cast<long long>(kPlanMinChunk), min(share, avg));
  auto chunks_of = [&](int n) -> int { return n > 2 * L ? static_cast<int>((n + L - 1) / L) : 1; };  // n >= 0
  // each thread takes a contiguous segment of units, in unit order
  const int seg = (units + kPlanThreads - 1) / kPlanThreads;
  const int u0 = min(units, tid * seg), u1 = min(units, u0 + seg);
  int items = 0, slots = 0, splits = 0, steps = 0;
  for (int u = u0; u < u1; ++u) {
    const int c = chunks_of(nbuf[u]);
    items += c;
    steps += nbuf[u];
    if (c > 1) {
      slots += c;
      ++splits;
    }
  }
  scan_items[tid] = items;
  scan_slots[tid] = slots;
  scan_splits[tid] = splits;
  scan_steps[tid] = steps;
  __syncthreads();
  if (tid == 0) {  // exclusive scans in segment (= unit) order; segments over the slot budget stay unsplit
    int ai = 0, as = 0, ap = 0, at = 0;
    for (int i = 0; i < kPlanThreads; ++i) {
      const int xt = scan_steps[i];
      scan_steps[i] = at;
      at += xt;
      int xi = scan_items[i], xs = scan_slots[i], xp = scan_splits[i];
      nosplit[i] = as + xs > max_slots;
      if (nosplit[i]) {
        xi = max(0, min(units, (i + 1) * seg) - min(units, i * seg));
        xs = 0;
        xp = 0;
      }
      scan_items[i] = ai;
      scan_slots[i] = as;
      scan_splits[i] = ap;
      ai += xi;
      as += xs;
      ap += xp;
    }
    a.plan[0] = ai;
    a.plan[1] = ap;
  }
  __syncthreads();
  int4* item = reinterpret_cast<int4*>(a.plan) + 1;
  int4* split = item + a.plan_max_items;
  int wi = scan_items[tid], ws = scan_slots[tid], wp = scan_splits[tid], wt = scan_steps[tid];
  for (int u = u0; u < u1; ++u) {
    const int n = nbuf[u];
    a.plan_sbase[u] = wt;
    if (n == 0) {  // nothing sees this key tile: one forced step, every score masked
      item[wi++] = make_int4(u, -1, 1, -1);
      continue;
    }
    const int c = nosplit[tid] ? 1 : chunks_of(n);
    const int per = (n + c - 1) / c;
    for (int k = 0; k < c; ++k)
      item[wi++] = make_int4(u, wt + k * per, min(per, n - k * per), c > 1 ? ws + k : -1);
    wt += n;
    if (c > 1) {
      split[wp++] = make_int4(u, ws, c, 0);
      ws += c;
    }
  }
}

// dV = sum of a split unit's chunk partials and dK = scale * sum, in chunk
// order, to bf16 (rows past the sequence are not written).
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_reduce_kernel(const BwdArgs a) {
  const int nsplit = a.plan[1];
  const int4* split = reinterpret_cast<const int4*>(a.plan) + 1 + a.plan_max_items;
  const int nlevels = (a.N + 127) / 128;
  const SeqSched sched{nullptr, a.nseq, a.N, a.Hkv, a.causal, nlevels, nullptr, 7};
  constexpr int kPer = 128 * D / 4;  // float4 per [128][D] tensor
  for (int sidx = blockIdx.x; sidx < nsplit; sidx += gridDim.x) {
    const int4 sp = split[sidx];
    const Unit un = decode_unit(sched, sp.x);
    for (int e = threadIdx.x; e < 2 * kPer; e += blockDim.x) {
      const int which = e / kPer, rem = e - which * kPer;
      const int row = rem / (D / 4), c4 = rem - row * (D / 4);
      const float4* src = reinterpret_cast<const float4*>(a.partials) + (static_cast<size_t>(sp.y) * 2 + which) * kPer + rem;
      float4 acc = src[0];
      for (int k = 1; k < sp.z; ++k) {
        const float4 x = src[static_cast<size_t>(k) * 2 * kPer];
        acc.x += x.x;
        acc.y += x.y;
        acc.z += x.z;
        acc.w += x.w;
      }
      const float mul = which == 0 ? 1.f : a.scale;
      const int key = un.qb2 * 128 + row;
      if (key < un.n) {
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(which == 0 ? a.dv : a.dk) +
                             (static_cast<size_t>(un.tok0 + key) * a.Hkv + un.h) * D + c4 * 4;
        *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(acc.x * mul, acc.y * mul), pack_bf16x2(acc.z * mul, acc.w * mul));
      }
    }
  }
}

// ------------------------------------------------------------------ block-sparse dQ rows
// The key blocks each (query head, query tile) row sees, as lists: counted
// (one warp per row, 32 mask bytes at a time), prefix-summed (one CTA), then
// written in order (ballot ranks). The dQ kernel reads block j of its row.
__device__ __forceinline__ int dq_row_end(const BwdArgs& a, int qt) { return a.causal ? min(a.nqb, qt + 1) : a.nqb; }

__global__ void __launch_bounds__(256) fa_bwd_rows_count_kernel(const BwdArgs a, int rows) {
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= rows) return;  // uniform over the warp
  const int qt = r % a.nqb, jend = dq_row_end(a, qt);
  const uint8_t* m = a.block_mask + static_cast<size_t>(r) * a.nqb;
  int n = 0;
  for (int base = 0; base < jend; base += 32)
    n += __popc(__ballot_sync(0xffffffffu, base + lane < jend && __ldg(m + base + lane) != 0));
  if (lane == 0) a.rows_n[r] = n;
}

__global__ void __launch_bounds__(kPlanThreads) fa_bwd_rows_scan_kernel(const BwdArgs a, int rows) {
  __shared__ int part[kPlanThreads];
  const int tid = threadIdx.x;
  const int seg = (rows + kPlanThreads - 1) / kPlanThreads;
  const int r0 = min(rows, tid * seg), r1 = min(rows, r0 + seg);
  int sum = 0;
  for (int r = r0; r < r1; ++r) sum += a.rows_n[r];
  part[tid] = sum;
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int i = 0; i < kPlanThreads; ++i) {
      const int x = part[i];
      part[i] = acc;
      acc += x;
    }
  }
  __syncthreads();
  int acc = part[tid];
  for (int r = r0; r < r1; ++r) {
    a.rows_base[r] = acc;
    acc += a.rows_n[r];
  }
}

__global__ void __launch_bounds__(256) fa_bwd_rows_list_kernel(const BwdArgs a, int rows) {
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= rows) return;  // uniform over the warp
  const int qt = r % a.nqb, jend = dq_row_end(a, qt);
  const uint8_t* m = a.block_mask + static_cast<size_t>(r) * a.nqb;
  int pos = a.rows_base[r];
  for (int base = 0; base < jend; base += 32) {
    const bool on = base + lane < jend && __ldg(m + base + lane) != 0;
    const uint32_t bal = __ballot_sync(0xffffffffu, on);
    if (on) a.rows_list[pos + __popc(bal & ((1u << lane) - 1u))] = base + lane;
    pos += __popc(bal);
  }
}

}  // namespace fa
