// Forward pass of exact attention on sm_100a: bf16 in, or fp8-e4m3 in with
// per-(head, 128-row block) scales (FA-3 summary, contribution 3: FP8 GEMMs);
// fp32 accumulation in both.
//
// What it computes: O = softmax(scale * Q K^T + mask) V and the per-row
// natural-log LSE, tile by tile, the score matrix living only in tensor
// memory (catalogue record "Dao and colleagues: IO-aware exact attention with
// FlashAttention", summary: exact attention without materialising the full
// attention matrix; Dao-AILab repository overview: online softmax with
// rescaling, tiled attention, persistent tile schedulers).
//
// Design (one persistent CTA per SM, 576 threads; 640 for fp8):
//   warps 0-7   softmax of query tile 0: warp w takes TMEM lanes (rows)
//               32*(w%4).. and key columns 64*((w/4)%2)..; the two warps of
//               a row quadrant exchange row maxima and sums through smem at
//               a named barrier of their own
//   warps 8-15  softmax of query tile 1, likewise
//   warp  16    TMA producer: Q tiles once per unit, K_j / V_j through a ring
//   warp  17    tcgen05 issuer (one thread) and TMEM owner
//   warps 18-19 fp8 only: widen e4m3 V tiles to f16
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [384,384+D).
// P (bf16) is written over the first 64 columns of its S tile and fed to the
// PV MMA straight from TMEM. The two query tiles ping-pong: while one tile's
// softmax runs, the tensor core works on the other tile's GEMMs.
#pragma once

#include "fa_tile.cuh"

namespace fa {

// Warp roles: 16 softmax warps (two per TMEM lane quadrant per query tile,
// each on one half of the 128 key columns), the TMA producer, the MMA
// issuer; fp8 adds two warps that widen each e4m3 V tile to f16.
constexpr int kSoftmaxWarps = 16;
constexpr int kWarpProducer = 16;
constexpr int kWarpMma = 17;
constexpr int kWarpConv = 18;
constexpr int kThreadsFwd = 18 * 32;
constexpr int kThreadsFwdF8 = 20 * 32;
constexpr float kTau = 8.0f;  // lazy-rescale threshold, base-2 exponent units
// Named barrier of the two softmax warps that share a query tile's TMEM lane
// quadrant (ids 1..8; 0 is __syncthreads)
__host__ __device__ constexpr int fwd_pair_barrier(int tile, int quad) { return 1 + tile * 4 + quad; }


struct FwdArgs {
  void* o;
  float* lse;
  const int* cu_seqlens;
  int nseq;        // padded: B
  int N;           // padded: N; varlen: max_seqlen
  int total_T;     // tokens in the packed token dimension
  int Hq, Hkv;
  int causal;
  float scale;     // softmax scale
  float scale_log2;  // scale * log2(e)
  int lse_head_stride;  // padded: N; varlen: total_T
  int num_units;   // padded: exact; varlen: upper bound
  uint64_t timeout_ns;
  int* status;
  int inject;      // test hook: 1 = the producer never loads the first K tile
  // block-sparse: [Hq][nqb][nqb] uint8, key block j visible to query block i
  // of head h when nonzero (shared by the batch); null = dense
  const uint8_t* block_mask;
  int nqb;
  // fp8 only: block scales [B, H, nblk_s] (value = code * scale)
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
  int nblk_s;
};

template <int D, int STAGES, bool F8 = false>
struct FwdSmem {
  static constexpr int kTileBytes = kBM * D * (F8 ? 1 : 2);  // one 128 x D tile
  alignas(1024) uint8_t q[2][kTileBytes];
  alignas(1024) uint8_t kv[STAGES][kTileBytes];
  // fp8: V tiles widened to f16 (exact), double-buffered
  static constexpr int kV16Bytes = F8 ? kBM * D * 2 : 1024;
  alignas(1024) uint8_t v16[2][kV16Bytes];
  uint64_t q_full, q_empty;
  uint64_t kv_full[STAGES], kv_empty[STAGES];
  uint64_t s_full[2], p_full[2], o_final[2], o_free[2];
  uint64_t v16_full[2], v16_empty[2];
  float xch[2][2][2][128];        // [slot][tile][half][row] values exchanged by a pair
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int level_count[512];
};

// O += P V: P (bf16 or f16 pairs) read from TMEM in the split layout above,
// V a [keys, D] tile (D contiguous) in shared memory as the MN-major B
// operand: LBO = next 64 columns of D (next 16 KB box), SBO = next 8 keys.
// One MMA covers 16 keys.
template <int D, bool F16 = false>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_smem, bool accumulate) {
  constexpr uint32_t idesc = F16 ? idesc_f16_f32(kBM, D, false, true) : idesc_bf16_f32(kBM, D, false, true);
  const uint64_t vd = smem_desc(v_smem, 16384, 1024, kSwizzle128B);
  const uint32_t acc0 = accumulate ? 1u : 0u;
#pragma unroll
  for (int kk = 0; kk < kBN / 16; ++kk)
    mma_f16_ts(o_tmem, p_tmem + split_a_col(kk), vd + static_cast<uint64_t>((kk * 2048) >> 4), idesc,
               kk > 0 ? 1u : acc0);
}

// fp8: widens `nkeys` rows (keys) of an e4m3 V tile to f16 (exactly) in the
// 128B-swizzled MN-major layout the PV MMA reads; thread t of nthreads takes
// every nthreads-th (key, 16-element chunk). `src` and `dst` point at the
// first row handled (a multiple of 8 rows into the tile).
template <int D>
__device__ __forceinline__ void widen_v_tile(const uint8_t* src, uint8_t* dst, int t, int nthreads, int nkeys) {
  static_assert(D == 128, "fp8 path is built for d = 128");
  for (int u = t; u < nkeys * 8; u += nthreads) {
    const int r = u >> 3;      // key
    const int c16 = u & 7;     // 16-element (16-byte) chunk of the e4m3 row
    const uint4 v = *reinterpret_cast<const uint4*>(src + r * 128 + ((c16 ^ (r & 7)) << 4));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t h[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      h[2 * i] = e4m3x2_to_f16x2(static_cast<uint16_t>(w[i] & 0xffffu));
      h[2 * i + 1] = e4m3x2_to_f16x2(static_cast<uint16_t>(w[i] >> 16));
    }
    // elements 16*c16 .. +15 -> f16 box c16/4, 8-element chunks 2*(c16%4), +1
    uint8_t* box = dst + (c16 >> 2) * 16384 + r * 128;
    const int c8 = 2 * (c16 & 3);
    *reinterpret_cast<uint4*>(box + ((c8 ^ (r & 7)) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4*>(box + (((c8 + 1) ^ (r & 7)) << 4)) = make_uint4(h[4], h[5], h[6], h[7]);
  }
}

// 4 x 4 transpose of 16-byte pieces over the four lanes l = 4g..4g+3: on
// entry lane l holds pieces (row l, piece c) in p[c]; on exit it holds
// (row 4g + c, piece l % 4) in p[c]. Two stages; in stage b a lane swaps,
// with lane l ^ b, the pieces whose bit b differs from its own lane bit.
__device__ __forceinline__ void transpose4_pieces(uint4 (&p)[4], int lane) {
#pragma unroll
  for (int b = 1; b <= 2; b <<= 1) {
    const bool hi = lane & b;
#pragma unroll
    for (int c0 = 0; c0 < 4; ++c0) {
      if (c0 & b) continue;
      const int c1 = c0 | b;
      const uint4 send = hi ? p[c0] : p[c1];
      uint4 r;
      r.x = __shfl_xor_sync(0xffffffffu, send.x, b);
      r.y = __shfl_xor_sync(0xffffffffu, send.y, b);
      r.z = __shfl_xor_sync(0xffffffffu, send.z, b);
      r.w = __shfl_xor_sync(0xffffffffu, send.w, b);
      if (hi)
        p[c0] = r;
      else
        p[c1] = r;
    }
  }
}

__device__ __forceinline__ int num_kv_blocks(const Unit& u, int causal) {
  const int nb = (u.n + kBN - 1) / kBN;
  return causal ? min(nb, 2 * u.qb2 + 2) : nb;
}

// Block-sparse walk over the key blocks [0, jend) of a unit (query blocks
// qb0, qb0 + 1 of head h): a block is visited when either query block may see
// it. A unit whose query blocks see no key block still visits block 0, with
// every score masked (O = 0, LSE = -inf), so that every role runs the same
// pipeline. Without a mask every block is visited.
__device__ __forceinline__ bool kv_block_on(const FwdArgs& a, int h, int qb, int j) {
  return qb < a.nqb && __ldg(a.block_mask + (static_cast<size_t>(h) * a.nqb + qb) * a.nqb + j) != 0;
}
// Bit e set when key block base + e (< jend) is seen by query block qb0 or
// qb0 + 1: eight independent loads per round, one round trip for eight
// blocks (the mask is read through L2).
__device__ __forceinline__ uint32_t kv_blocks_on8(const FwdArgs& a, int h, int qb0, int base, int jend) {
  const uint8_t* r0 = a.block_mask + (static_cast<size_t>(h) * a.nqb + qb0) * a.nqb;
  const bool has1 = qb0 + 1 < a.nqb;
  uint32_t on = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int jj = base + e;
    const uint8_t x0 = jj < jend ? __ldg(r0 + jj) : 0;
    const uint8_t x1 = jj < jend && has1 ? __ldg(r0 + a.nqb + jj) : 0;
    on |= (x0 | x1) ? (1u << e) : 0u;
  }
  return on;
}
__device__ __forceinline__ int next_kv_block(const FwdArgs& a, int h, int qb0, int j, int jend) {
  if (a.block_mask == nullptr) return j + 1;
  for (int base = j + 1; base < jend; base += 8) {
    const uint32_t on = kv_blocks_on8(a, h, qb0, base, jend);
    if (on) return base + __ffs(on) - 1;
  }
  return jend;
}
__device__ __forceinline__ int first_kv_block(const FwdArgs& a, int h, int qb0, int jend) {
  const int j = next_kv_block(a, h, qb0, -1, jend);
  return j < jend ? j : 0;
}
__device__ __forceinline__ int count_kv_blocks(const FwdArgs& a, int h, int qb0, int jend) {
  if (a.block_mask == nullptr) return jend;
  int n = 0;
  for (int base = 0; base < jend; base += 8) n += __popc(kv_blocks_on8(a, h, qb0, base, jend));
  return n > 0 ? n : 1;
}

// The softmax warps' copy of a unit's two mask rows: lane i holds, in bit e
// of rows[t], whether query block qb0 + t sees key block 32 i + e (< jend).
// Loaded once per unit (64 independent byte loads per lane, one round trip);
// the walk over visible blocks and the per-tile flags are then warp
// operations on registers. nqb <= 1024 (32 blocks per lane).
struct WarpMaskRows {
  uint32_t rows[2];
};
__device__ __forceinline__ WarpMaskRows warp_mask_rows(const FwdArgs& a, int h, int qb0, int jend, int lane) {
  WarpMaskRows w{{0u, 0u}};
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    if (qb0 + t >= a.nqb) continue;
    const uint8_t* r = a.block_mask + (static_cast<size_t>(h) * a.nqb + qb0 + t) * a.nqb;
    uint8_t x[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) x[e] = lane * 32 + e < jend ? __ldg(r + lane * 32 + e) : 0;
#pragma unroll
    for (int e = 0; e < 32; ++e) w.rows[t] |= x[e] ? (1u << e) : 0u;
  }
  return w;
}
// First visible block (either tile) after j, or jend; warp-uniform.
__device__ __forceinline__ int warp_next_block(const WarpMaskRows& w, int j, int jend, int lane) {
  const int from = j + 1;
  uint32_t word = w.rows[0] | w.rows[1];
  if (lane * 32 + 31 < from)
    word = 0;
  else if (lane * 32 < from)
    word &= ~((1u << (from - lane * 32)) - 1u);
  const uint32_t bal = __ballot_sync(0xffffffffu, word != 0);
  if (bal == 0) return jend;
  const int src = __ffs(bal) - 1;
  const uint32_t ws = __shfl_sync(0xffffffffu, word, src);
  return src * 32 + __ffs(ws) - 1;
}
__device__ __forceinline__ int warp_count_blocks(const WarpMaskRows& w) {
  return __reduce_add_sync(0xffffffffu, __popc(w.rows[0] | w.rows[1]));
}
__device__ __forceinline__ bool warp_tile_on(const WarpMaskRows& w, int tile, int jb) {
  return (__shfl_sync(0xffffffffu, w.rows[tile], jb >> 5) >> (jb & 31)) & 1u;
}

// Exponentials of 2*NP consecutive columns of one row: p = 2^(s*cj - m),
// packed in pairs (bf16, or f16 of p*pmul on the fp8 path) into pk[NP] for
// the PV MMA; returns the fp32 sum. Scale and sum run on packed fp32 pairs,
// the exponentials on the MUFU unit.
template <bool F16, int NP = 32>
__device__ __forceinline__ float exp_pack(const float* s, float cj, float m, float pmul, uint32_t* pk) {
  const uint64_t c2 = f2(cj, cj);
  const uint64_t nm2 = f2(-m, -m);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int t = 0; t < NP; ++t) {
    const uint64_t x2 = f2_fma(f2(s[2 * t], s[2 * t + 1]), c2, nm2);
    const float2 x = f2_split(x2);
    const float p0 = ex2_approx(x.x);
    const float p1 = ex2_approx(x.y);
    acc[t & 3] = f2_add(acc[t & 3], f2(p0, p1));
    if constexpr (F16)
      pk[t] = pack_f16x2(p0 * pmul, p1 * pmul);
    else
      pk[t] = pack_bf16x2(p0, p1);
  }
  const float2 a = f2_split(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])));
  return a.x + a.y;
}

template <int D, int STAGES, bool F8, bool SPARSE = false>
__global__ void __launch_bounds__(F8 ? kThreadsFwdF8 : kThreadsFwd, 1)
    fa_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const FwdArgs args) {
  using Smem = FwdSmem<D, STAGES, F8>;
  constexpr int EB = F8 ? 1 : 2;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // ---- set-up: barriers, TMEM, varlen level table
  if (tid == 0) {
    mbar_init(smem_u32(&sm.q_full), 1);
    mbar_init(smem_u32(&sm.q_empty), 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&sm.kv_full[s]), 1);
      mbar_init(smem_u32(&sm.kv_empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.s_full[i]), 1);
      mbar_init(smem_u32(&sm.p_full[i]), 8);  // one arrival per softmax warp of the tile
      mbar_init(smem_u32(&sm.o_final[i]), 1);
      mbar_init(smem_u32(&sm.o_free[i]), 8);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.v16_full[i]), 2);  // one arrival per converter warp
      mbar_init(smem_u32(&sm.v16_empty[i]), 1);
    }
    if constexpr (F8) {
      // V tiles sit in the odd ring slots and are released by the two
      // converter warps instead of an MMA commit
      for (int s = 1; s < STAGES; s += 2) mbar_init(smem_u32(&sm.kv_empty[s]), 2);
    }
    mbar_init(smem_u32(&sm.drain), 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  constexpr int kThreads = F8 ? kThreadsFwdF8 : kThreadsFwd;
  const int nlevels = (args.N + 255) / 256;
  const bool varlen = args.cu_seqlens != nullptr;
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(&sm.tmem_base), 512);
    tmem_relinquish();
  }
  if (warp == kWarpProducer && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  __syncthreads();
  int num_units = args.num_units;
  if (varlen)
    num_units = varlen_level_table(sm.level_count, args.cu_seqlens, args.nseq, nlevels, 8, args.Hq, kThreads);
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  SeqSched sched{args.cu_seqlens, args.nseq, args.N, args.Hq, !args.causal, nlevels, sm.level_count, 8,
                 !SPARSE && !varlen && !args.causal};
  const volatile int* abort = &sm.abort;
  const int group = args.Hq / args.Hkv;
  uint32_t prod_issued = 0;  // K/V loads issued by the producer thread
  uint32_t q_issued = 0;     // Q loads issued by the producer thread

  if (warp == kWarpProducer) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      uint32_t kv_prod = 0, it = 0;
      bool ok = true;
      for (int rnd = 0; ok; ++rnd, ++it) {
        const int u = unit_of(rnd, blockIdx.x, gridDim.x);
        if (u >= num_units) break;
        const Unit un = decode_unit(sched, u);
        const int jend = num_kv_blocks(un, args.causal);
        const int nblk = SPARSE ? count_kv_blocks(args, un.h, un.qb2 * 2, jend) : jend;
        const int hkv = un.h / group;
        if (!mbar_wait(smem_u32(&sm.q_empty), (it & 1) ^ 1, abort, args.timeout_ns)) {
          report_error(args.status, kStatusTimeout, 1);
          ok = false;
          break;
        }
        const uint32_t qbar = smem_u32(&sm.q_full);
        mbar_expect_tx(qbar, 2 * Smem::kTileBytes);
        const int row0 = un.tok0 + un.qb2 * 2 * kBM;
        load_tile<D, EB>(smem_u32(sm.q[0]), &tm_q, qbar, un.h, row0);
        load_tile<D, EB>(smem_u32(sm.q[1]), &tm_q, qbar, un.h, row0 + kBM);
        q_issued = it + 1;
        int jb = SPARSE ? first_kv_block(args, un.h, un.qb2 * 2, jend) : 0;  // key block of the j-th visit
        for (int j = 0; j < nblk && ok; ++j, jb = SPARSE ? next_kv_block(args, un.h, un.qb2 * 2, jb, jend) : jb + 1) {
          for (int kv = 0; kv < 2; ++kv) {
            const uint32_t slot = kv_prod % STAGES;
            if (!mbar_wait(smem_u32(&sm.kv_empty[slot]), ((kv_prod / STAGES) & 1) ^ 1, abort, args.timeout_ns)) {
              report_error(args.status, kStatusTimeout, 2);
              ok = false;
              break;
            }
            if (args.inject == 1 && it == 0 && j == 0 && kv == 0) {
              // test hook: the first K tile of the unit is never loaded
            } else {
              const uint32_t bar = smem_u32(&sm.kv_full[slot]);
              mbar_expect_tx(bar, Smem::kTileBytes);
              load_tile<D, EB>(smem_u32(sm.kv[slot]), kv == 0 ? &tm_k : &tm_v, bar, hkv, un.tok0 + jb * kBN);
            }
            ++kv_prod;
          }
        }
      }
      if (!ok) sm.abort = 1;
      prod_issued = kv_prod;
    }
  } else if (warp == kWarpMma) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      uint32_t kv_cons = 0, it = 0, pc0 = 0, pc1 = 0, g = 0;
      bool ok = true;
      const uint32_t S0 = tmem + 0, S1 = tmem + 128, O0 = tmem + 256, O1 = tmem + 384;
      auto wait = [&](uint64_t* bar, uint32_t parity, int site) -> bool {
        if (!mbar_wait(smem_u32(bar), parity, abort, args.timeout_ns)) {
          report_error(args.status, kStatusTimeout, site);
          return false;
        }
        tc_fence_after();
        return true;
      };
      for (int rnd = 0; ok; ++rnd, ++it) {
        const int u = unit_of(rnd, blockIdx.x, gridDim.x);
        if (u >= num_units) break;
        const Unit un = decode_unit(sched, u);
        const int nblk =
            SPARSE ? count_kv_blocks(args, un.h, un.qb2 * 2, num_kv_blocks(un, args.causal)) : num_kv_blocks(un, args.causal);
        if (!(ok = wait(&sm.q_full, it & 1, 10))) break;
        const uint32_t q0 = smem_u32(sm.q[0]), q1 = smem_u32(sm.q[1]);
        uint32_t slotK = kv_cons % STAGES;
        if (!(ok = wait(&sm.kv_full[slotK], (kv_cons / STAGES) & 1, 11))) break;
        ++kv_cons;
        issue_qk<D, F8>(S0, q0, smem_u32(sm.kv[slotK]));
        tc_commit(smem_u32(&sm.s_full[0]));
        issue_qk<D, F8>(S1, q1, smem_u32(sm.kv[slotK]));
        tc_commit(smem_u32(&sm.s_full[1]));
        tc_commit(smem_u32(&sm.kv_empty[slotK]));
        if (nblk == 1) tc_commit(smem_u32(&sm.q_empty));
        for (int j = 0; j < nblk; ++j, ++g) {
          const bool has_next = j + 1 < nblk;
          const uint32_t slotV = kv_cons % STAGES;
          if constexpr (F8) {
            if (!(ok = wait(&sm.v16_full[g & 1], (g >> 1) & 1, 18))) break;
          } else {
            if (!(ok = wait(&sm.kv_full[slotV], (kv_cons / STAGES) & 1, 12))) break;
          }
          ++kv_cons;
          if (has_next) {
            slotK = kv_cons % STAGES;
            if (!(ok = wait(&sm.kv_full[slotK], (kv_cons / STAGES) & 1, 13))) break;
            ++kv_cons;
          }
          const uint32_t vaddr = F8 ? smem_u32(sm.v16[g & 1]) : smem_u32(sm.kv[slotV]);
          // ---- tile 0
          if (!(ok = wait(&sm.p_full[0], pc0 & 1, 14))) break;
          ++pc0;
          if (j == 0 && !(ok = wait(&sm.o_free[0], (it & 1) ^ 1, 15))) break;
          issue_pv<D, F8>(O0, S0, vaddr, j > 0);
          if (has_next) {
            issue_qk<D, F8>(S0, q0, smem_u32(sm.kv[slotK]));
            tc_commit(smem_u32(&sm.s_full[0]));
          } else {
            tc_commit(smem_u32(&sm.o_final[0]));
          }
          // ---- tile 1
          if (!(ok = wait(&sm.p_full[1], pc1 & 1, 16))) break;
          ++pc1;
          if (j == 0 && !(ok = wait(&sm.o_free[1], (it & 1) ^ 1, 17))) break;
          issue_pv<D, F8>(O1, S1, vaddr, j > 0);
          tc_commit(F8 ? smem_u32(&sm.v16_empty[g & 1]) : smem_u32(&sm.kv_empty[slotV]));
          if (has_next) {
            issue_qk<D, F8>(S1, q1, smem_u32(sm.kv[slotK]));
            tc_commit(smem_u32(&sm.s_full[1]));
            tc_commit(smem_u32(&sm.kv_empty[slotK]));
            if (j + 2 == nblk) tc_commit(smem_u32(&sm.q_empty));
          } else {
            tc_commit(smem_u32(&sm.o_final[1]));
          }
        }
      }
      if (!ok) sm.abort = 1;
      // every MMA issued so far must finish before TMEM is released
      tc_commit(smem_u32(&sm.drain));
      mbar_wait(smem_u32(&sm.drain), 0, nullptr, args.timeout_ns);
    }
  } else if (warp >= kWarpConv) {
    // ======================= fp8: V widening warps =======================
    if constexpr (F8) {
      const int t = tid - kWarpConv * 32;
      uint32_t g = 0, it = 0;
      bool ok = true;
      for (int rnd = 0; ok; ++rnd, ++it) {
        const int u = unit_of(rnd, blockIdx.x, gridDim.x);
        if (u >= num_units) break;
        const Unit un = decode_unit(sched, u);
        const int nblk =
            SPARSE ? count_kv_blocks(args, un.h, un.qb2 * 2, num_kv_blocks(un, args.causal)) : num_kv_blocks(un, args.causal);
        for (int j = 0; j < nblk; ++j, ++g) {
          const uint32_t idx = 2 * g + 1;  // ring index of V_j (K and V alternate)
          const uint32_t slot = idx % STAGES;
          ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.kv_full[slot]), (idx / STAGES) & 1, abort,
                                                 args.timeout_ns));
          if (ok)
            ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.v16_empty[g & 1]), ((g >> 1) & 1) ^ 1, abort,
                                                   args.timeout_ns));
          if (!ok) {
            if (lane == 0) report_error(args.status, kStatusTimeout, 25);
            break;
          }
          // converter warp c widens keys 64*c .. +63
          widen_v_tile<D>(sm.kv[slot] + (warp - kWarpConv) * 64 * 128, sm.v16[g & 1] + (warp - kWarpConv) * 64 * 128, lane,
                          32, 64);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(smem_u32(&sm.v16_full[g & 1]));
            mbar_arrive(smem_u32(&sm.kv_empty[slot]));
          }
        }
      }
      if (!ok) sm.abort = 1;
      (void)t;
    }
  } else if (warp < kSoftmaxWarps) {
    // ======================= softmax warps =======================
    // warp w: query tile w/8, TMEM lane quadrant w%4 (row = lane), key column
    // half (w/4)%2 of every 128-column S block
    const int tile = warp >> 3;
    const int quad = warp & 3;
    const int half = (warp >> 2) & 1;
    const int r_in_tile = quad * 32 + lane;
    const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t S = tmem + tile * 128 + 64 * half + lane_bits;          // this half of S
    constexpr int HC = D / 2;                                              // O columns per half
    const uint32_t O = tmem + 256 + tile * 128 + HC * half + lane_bits;    // this half of O
    const int pair_bar = fwd_pair_barrier(tile, quad);
    const float cl = args.scale_log2;
    constexpr float tau = kTau;
    uint32_t sc = 0, xc = 0, it = 0;
    bool ok = true;
    // Hands v to the partner warp (same rows, other column half) and returns
    // its value: a barrier over the pair's 64 threads that also ORs their
    // failure flags, so both warps leave together and neither waits at the
    // barrier for a partner that has gone. Two smem slots alternate: a warp
    // writes slot s again only after the partner has passed the barrier that
    // follows its read of slot s.
    auto exchange = [&](bool good, float v, float& other) -> bool {
      const int slot = xc & 1;
      if (good) sm.xch[slot][tile][half][r_in_tile] = v;
      const bool fail = bar_red_or(!good, pair_bar, 64);
      ++xc;
      other = sm.xch[slot][tile][half ^ 1][r_in_tile];
      return !fail;
    };
    for (int rnd = 0; ok; ++rnd, ++it) {
      const int u = unit_of(rnd, blockIdx.x, gridDim.x);
      if (u >= num_units) break;
      const Unit un = decode_unit(sched, u);
      const int jend = num_kv_blocks(un, args.causal);
      WarpMaskRows wm{{0u, 0u}};
      if constexpr (SPARSE) wm = warp_mask_rows(args, un.h, un.qb2 * 2, jend, lane);
      int nblk = jend;  // key blocks visited (block-sparse: at least one, block 0 fully masked)
      if constexpr (SPARSE) nblk = max(warp_count_blocks(wm), 1);
      const int row = un.qb2 * 2 * kBM + tile * kBM + r_in_tile;  // row within the sequence
      const int limit = args.causal ? min(row, un.n - 1) : un.n - 1;  // last visible key
      // scores are kept in base-2 units t = s * cj; cj = scale*log2(e) for
      // bf16, times the query and key block scales for fp8
      float sq = 1.f, sv_max = 1.f;
      size_t kvs = 0;
      if constexpr (F8) {
        const int qt = un.qb2 * 2 + tile;
        if (qt < args.nblk_s) sq = args.q_scale[(static_cast<size_t>(un.seq) * args.Hq + un.h) * args.nblk_s + qt];
        kvs = (static_cast<size_t>(un.seq) * args.Hkv + un.h / group) * args.nblk_s;
        sv_max = 0.f;
        for (int jj = 0; jj < jend; ++jj) sv_max = fmaxf(sv_max, args.v_scale[kvs + jj]);
        sv_max = fmaxf(sv_max, 1e-30f);
      }
      float m = -INFINITY, l = 0.f;  // l: this half's share of the row sum
      int jb = 0;  // key block of the j-th visit
      if constexpr (SPARSE) {
        jb = warp_next_block(wm, -1, jend, lane);
        if (jb >= jend) jb = 0;
      }
      for (int j = 0; j < nblk; ++j, jb = SPARSE ? warp_next_block(wm, jb, jend, lane) : jb + 1) {
        float cj = cl, pmul = 1.f;
        if constexpr (F8) {
          cj = cl * sq * args.k_scale[kvs + jb];
          pmul = args.v_scale[kvs + jb] / sv_max;
        }
        // every lane waits; the outcome is made warp-uniform so that the
        // warp-collective tcgen05 loads below run converged, and is shared
        // with the partner warp at the exchange
        const bool good =
            __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.s_full[tile]), sc & 1, abort, args.timeout_ns));
        ++sc;
        const int kv0 = jb * kBN + 64 * half;  // first key of this half
        // block-sparse: the whole block is hidden from this tile (uniform over the tile)
        const bool tile_on = !SPARSE || warp_tile_on(wm, tile, jb);
        // warp-uniform: every lane of a warp takes the same masked/unmasked path
        const bool masked_blk = !tile_on || __any_sync(0xffffffffu, kv0 + 63 > limit);
        // pass 1: this half's row maximum, exchanged with the partner half
        float pm = -INFINITY;
        if (good) {
          uint32_t sr[64];
          float* sv = reinterpret_cast<float*>(sr);
          tc_fence_after();
          tmem_ld64(S, sr);
          if (masked_blk) {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (!tile_on || kv0 + c > limit) sv[c] = -INFINITY;
          }
          float a = fmax3(sv[0], sv[1], sv[2]);
          float b = fmax3(sv[32], sv[33], sv[34]);
#pragma unroll
          for (int c = 3; c < 31; c += 2) {
            a = fmax3(a, sv[c], sv[c + 1]);
            b = fmax3(b, sv[32 + c], sv[32 + c + 1]);
          }
          pm = fmax3(fmaxf(a, sv[31]), b, sv[63]);
        }
        float po;
        if (!exchange(good, pm, po)) {
          ok = false;
          if (!good && lane == 0) report_error(args.status, kStatusTimeout, 20 + tile);
          break;
        }
        const float mt = fmaxf(pm, po) * cj;  // identical in both halves
        const bool need = mt - m > tau;
        const float m_new = need ? mt : m;
        const float alpha = need ? ex2_approx(m - m_new) : 1.f;
        if (j > 0 && __any_sync(0xffffffffu, need)) {
          // this half's O columns are rescaled in TMEM; the PV MMA of the
          // previous block has completed (it precedes this S in issue order)
#pragma unroll 1
          for (int c = 0; c < HC; c += 32) {
            uint32_t orr[32];
            tmem_ld32(O + c, orr);
#pragma unroll
            for (int t = 0; t < 32; ++t) orr[t] = __float_as_uint(__uint_as_float(orr[t]) * alpha);
            tmem_st32(O + c, orr);
          }
        }
        // pass 2: P = 2^(s*cj - m) in two 32-column chunks; chunk c's P pairs
        // go to columns [16c, 16c+16) of this half, already read
        float lsum = 0.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t sr[32];
          tmem_ld32(S + 32 * c, sr);
          float* sv = reinterpret_cast<float*>(sr);
          if (masked_blk) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (!tile_on || kv0 + 32 * c + e > limit) sv[e] = -INFINITY;
          }
          uint32_t pk[16];
          // a row that has seen no visible key yet (block-sparse) keeps
          // m = -inf: its exponentials are taken against 0 and are all 0
          lsum += masked_blk ? exp_pack<F8, 16>(sv, cj, SPARSE && m_new == -INFINITY ? 0.f : m_new, pmul, pk)
                             : exp_pack<F8, 16>(sv, cj, m_new, pmul, pk);
          tmem_st16(S + 16 * c, pk);
        }
        l = l * alpha + lsum;
        m = m_new;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.p_full[tile]));
      }
      if (!ok) break;
      // ---- epilogue: O / l -> bf16 (this half's columns), LSE
      const bool good =
          __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.o_final[tile]), it & 1, abort, args.timeout_ns));
      float lo;
      if (!exchange(good, l, lo)) {
        ok = false;
        if (!good && lane == 0) report_error(args.status, kStatusTimeout, 22 + tile);
        break;
      }
      tc_fence_after();
      const float lt = l + lo;
      const bool valid = row < un.n;
      // fp8: P entered the PV MMA scaled by sv_j / sv_max
      const float inv_l = !SPARSE || lt > 0.f ? (F8 ? sv_max : 1.f) / lt : 0.f;  // no visible key: O = 0
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(args.o) +
                            (static_cast<size_t>(un.tok0 + row) * args.Hq + un.h) * D + HC * half;
#pragma unroll 1
      for (int c = 0; c < HC; c += 32) {
        uint32_t orr[32];
        tmem_ld32(O + c, orr);
        uint32_t pk[16];
#pragma unroll
        for (int t = 0; t < 16; ++t)
          pk[t] = pack_bf16x2(__uint_as_float(orr[2 * t]) * inv_l, __uint_as_float(orr[2 * t + 1]) * inv_l);
        // each lane holds four 16-byte pieces of its row; a 4 x 4 transpose
        // over the four lanes of consecutive rows (two xor stages of
        // shuffles) lets each store instruction write 64 contiguous bytes of
        // each of 8 rows instead of 16 bytes of each of 32
        uint4 pc[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) pc[t] = make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
        transpose4_pieces(pc, lane);
        const int j = lane & 3;
#pragma unroll
        for (int t = 0; t < 4; ++t)
          if (row - j + t < un.n)
            *reinterpret_cast<uint4*>(orow + static_cast<ptrdiff_t>(t - j) * args.Hq * D + c + 8 * j) = pc[t];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.o_free[tile]));
      if (valid && half == 0) {
        const size_t li = varlen ? (static_cast<size_t>(un.h) * args.lse_head_stride + un.tok0 + row)
                                 : (static_cast<size_t>(un.seq * args.Hq + un.h) * args.lse_head_stride + row);
        // one explicit fused multiply-add: every instantiation rounds the LSE alike
        args.lse[li] = !SPARSE || lt > 0.f ? __fmaf_rn(m, 0.6931471805599453f, logf(lt)) : -INFINITY;
      }
    }
    if (!ok) sm.abort = 1;
  }

  // ---- teardown: every role is out of its loop; release TMEM
  tc_fence_before();
  __syncthreads();
  if (sm.abort && warp == kWarpProducer && lane == 0) {
    // after an abort, let the K/V loads already issued land before the CTA
    // exits (the newest load of each ring slot is the one still in flight)
    for (uint32_t i = (prod_issued > STAGES ? prod_issued - STAGES : 0); i < prod_issued; ++i) {
      if (args.inject == 1 && i == 0) continue;  // never issued
      mbar_wait(smem_u32(&sm.kv_full[i % STAGES]), (i / STAGES) & 1, nullptr, args.timeout_ns);
    }
    if (q_issued > 0) mbar_wait(smem_u32(&sm.q_full), (q_issued - 1) & 1, nullptr, args.timeout_ns);
  }
  __syncthreads();
  if (warp == kWarpMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa
