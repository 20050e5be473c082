// Preparation pass of the backward: D = rowsum(dO * O) (the term the
// softmax gradient subtracts, dS = P * (dP - D)) and the forward's LSE in
// base 2, per (token, query head), into the workspace the dK/dV and dQ
// kernels read.
#pragma once

#include "fa_bwd_args.cuh"

namespace fa {

// First token of sequence s (s = nseq: total_T).
__device__ __forceinline__ int seq_start(const BwdArgs& a, int s) {
  return a.cu_seqlens ? __ldg(a.cu_seqlens + s) : s * a.N;
}
// Sequence holding token t and t's row in it: padded, a division; packed, the
// last sequence that starts at or before t (a binary search over the starts;
// an empty sequence shares its start with the next one and is passed over).
__device__ __forceinline__ int token_seq(const BwdArgs& a, int t, int& row) {
  int s;
  if (a.cu_seqlens) {
    int lo = 0, hi = a.nseq - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(a.cu_seqlens + mid) <= t) lo = mid; else hi = mid - 1;
    }
    s = lo;
  } else {
    s = t / a.N;
  }
  row = t - seq_start(a, s);
  return s;
}

// D = dot(dO, O) in fp32 and the base-2 LSE for every token of every query
// head, then the filler values of the workspace gaps. O and dO are read as a
// stream of (token, head) entries in memory order, D*2 bytes each: a producer
// warp copies chunks of kPreChunk bytes of both into a ring of kPreStages
// shared-memory stages (cp.async.bulk, no registers held per byte in flight),
// and eight consumer warps reduce each entry with D/8 lanes (16 bytes a lane).
// Each consumer thread also owns one entry of the chunk for the output: it
// fetches the entry's LSE before waiting on the stage and writes LSE*log2(e)
// and D once the chunk's sums are in shared memory.
constexpr int kPreStages = 3;
constexpr int kPreChunk = 32768;  // bytes of O (and of dO) per stage
constexpr int kPreConsumers = 256;
constexpr int kPreThreads = kPreConsumers + 32;
struct PreSmem {
  alignas(128) uint8_t o[kPreStages][kPreChunk];
  alignas(128) uint8_t g[kPreStages][kPreChunk];
  float dsum[kPreStages][kPreConsumers];
  uint64_t full[kPreStages], empty[kPreStages];
  int consumed;
  int abort;
};

template <int D>
__global__ void __launch_bounds__(kPreThreads, 1) fa_bwd_pre_kernel(const BwdArgs a) {
  constexpr int EB = D * 2;            // bytes per entry
  constexpr int EC = kPreChunk / EB;   // entries per chunk (128 or 256)
  constexpr int LPR = D / 8;           // lanes per entry
  constexpr int EPW = 32 / LPR;        // entries per warp per pass
  static_assert(EC <= kPreConsumers && EC % (8 * EPW) == 0, "chunk layout");
  extern __shared__ uint8_t pre_raw[];
  PreSmem& sm = *reinterpret_cast<PreSmem*>((reinterpret_cast<uintptr_t>(pre_raw) + 127) & ~uintptr_t(127));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long total = static_cast<long long>(a.total_T) * a.Hq;
  const long long nchunks = (total + EC - 1) / EC;
  const volatile int* abort = &sm.abort;
  if (tid == 0) {
    for (int i = 0; i < kPreStages; ++i) {
      mbar_init(smem_u32(&sm.full[i]), 1);
      mbar_init(smem_u32(&sm.empty[i]), kPreConsumers / 32);
    }
    sm.consumed = 0;
    sm.abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  uint32_t issued = 0;
  if (warp == kPreConsumers / 32) {
    if (lane == 0) {
      const uint8_t* o = reinterpret_cast<const uint8_t*>(a.o);
      const uint8_t* g = reinterpret_cast<const uint8_t*>(a.dout);
      for (long long c = blockIdx.x; c < nchunks; c += gridDim.x, ++issued) {
        const uint32_t st = issued % kPreStages;
        if (!mbar_wait(smem_u32(&sm.empty[st]), ((issued / kPreStages) & 1) ^ 1, abort, a.timeout_ns)) {
          report_error(a.status, kStatusTimeout, 20);
          sm.abort = 1;
          break;
        }
        const long long e0 = c * EC;
        const uint32_t bytes = static_cast<uint32_t>(min(static_cast<long long>(EC), total - e0)) * EB;
        const uint32_t full = smem_u32(&sm.full[st]);
        mbar_expect_tx(full, 2 * bytes);
        bulk_load(smem_u32(sm.o[st]), o + e0 * EB, bytes, full);
        bulk_load(smem_u32(sm.g[st]), g + e0 * EB, bytes, full);
      }
    }
  } else {
    const int sub = lane / LPR, sl = lane % LPR;
    const bool narrow = total <= 0x7fffffffLL;  // 32-bit entry arithmetic
    // this thread's output entry of chunk c: its workspace index (or -1) and
    // its forward LSE, fetched one chunk ahead so that the load's latency
    // stays off the chunk's path
    auto entry_of = [&](long long c, long long& r, float& l) {
      r = -1;
      l = 0.f;
      const long long e = c * EC + tid;
      if (c >= nchunks || tid >= EC || e >= total) return;
      const int t = narrow ? static_cast<int>(static_cast<unsigned>(e) / static_cast<unsigned>(a.Hq))
                           : static_cast<int>(e / a.Hq);
      const int h = static_cast<int>(e - static_cast<long long>(t) * a.Hq);
      int row;
      const int seq = token_seq(a, t, row);
      const int t0 = seq_start(a, seq);
      const int idx = ws_offset(t0, seq) + row;
      // a token outside every sequence (cu_seqlens not covering [0, total_T)) has no entry
      if (row < 0 || row >= seq_start(a, seq + 1) - t0 || idx >= a.ws_stride) return;
      r = static_cast<long long>(h) * a.ws_stride + idx;
      const size_t li = a.cu_seqlens ? static_cast<size_t>(h) * a.lse_head_stride + t
                                     : (static_cast<size_t>(seq) * a.Hq + h) * a.lse_head_stride + row;
      l = __ldg(a.lse + li);
    };
    long long r_next;
    float l_next;
    entry_of(blockIdx.x, r_next, l_next);
    uint32_t k = 0;
    for (long long c = blockIdx.x; c < nchunks; c += gridDim.x, ++k) {
      const uint32_t st = k % kPreStages;
      const long long e0 = c * EC;
      const int n = static_cast<int>(min(static_cast<long long>(EC), total - e0));
      const long long r = r_next;
      const float l = l_next;
      entry_of(c + gridDim.x, r_next, l_next);
      bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.full[st]), (k / kPreStages) & 1, abort,
                                                   a.timeout_ns));
      if (ok) {
#pragma unroll 2
        for (int j = warp * EPW + sub; j < EC; j += (kPreConsumers / 32) * EPW) {
          float acc = 0.f;
          if (j < n) {
            const uint4 ov = *reinterpret_cast<const uint4*>(sm.o[st] + j * EB + sl * 16);
            const uint4 gv = *reinterpret_cast<const uint4*>(sm.g[st] + j * EB + sl * 16);
            const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
            const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const float2 x = __bfloat1622float2(o2[t]);
              const float2 y = __bfloat1622float2(g2[t]);
              acc = fmaf(x.x, y.x, acc);
              acc = fmaf(x.y, y.y, acc);
            }
          }
#pragma unroll
          for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
          if (sl == 0 && j < n) sm.dsum[st][j] = acc;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.empty[st]));  // the stage's bytes are read
      }
      // every consumer warp agrees (a timed-out wait on any ends them all); the
      // chunk's sums are in shared memory after this barrier
      ok = bar_red_and(ok, 1, kPreConsumers);
      if (!ok) {
        if (lane == 0) report_error(a.status, kStatusTimeout, 21);
        sm.abort = 1;
        break;
      }
      if (r >= 0) {
        // a row that saw no key (block-sparse: LSE = -inf) gets +inf, so P = 0
        a.lse2[r] = (l == -INFINITY ? INFINITY : l) * kLog2e;
        a.dvec[r] = sm.dsum[st][tid];
      }
      if (tid == 0) sm.consumed = static_cast<int>(k + 1);
    }
    // the gap after each sequence's rows (up to the next sequence's block; the
    // last one up to ws_stride; the first sequence also the entries before its
    // block): +inf (LSE) and 0 (D), one warp per (head, sequence)
    const long long ngaps = static_cast<long long>(a.Hq) * a.nseq;
    const int cw = kPreConsumers / 32;
    for (long long gi = static_cast<long long>(blockIdx.x) * cw + warp; gi < ngaps;
         gi += static_cast<long long>(gridDim.x) * cw) {
      const int h = static_cast<int>(gi / a.nseq);
      const int s = static_cast<int>(gi - static_cast<long long>(h) * a.nseq);
      const int t0 = seq_start(a, s), t1 = seq_start(a, s + 1);
      const int from = ws_offset(t0, s) + (t1 - t0);
      const int to = s + 1 < a.nseq ? ws_offset(t1, s + 1) : a.ws_stride;
      const int lead = s == 0 ? min(ws_offset(t0, 0), a.ws_stride) : 0;
      for (int i = lane; i < lead; i += 32) {
        a.lse2[static_cast<size_t>(h) * a.ws_stride + i] = INFINITY;
        a.dvec[static_cast<size_t>(h) * a.ws_stride + i] = 0.f;
      }
      for (int i = max(from, 0) + lane; i < min(to, a.ws_stride); i += 32) {
        const size_t ri = static_cast<size_t>(h) * a.ws_stride + i;
        a.lse2[ri] = INFINITY;
        a.dvec[ri] = 0.f;
      }
    }
  }
  __syncthreads();
  // after an abort, the copies issued but not consumed must land before the
  // CTA's shared memory is released
  if (sm.abort && warp == kPreConsumers / 32 && lane == 0) {
    for (uint32_t i = static_cast<uint32_t>(sm.consumed); i < issued; ++i)
      mbar_wait(smem_u32(&sm.full[i % kPreStages]), (i / kPreStages) & 1, nullptr, a.timeout_ns);
  }
}

}  // namespace fa
