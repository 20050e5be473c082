// Shared definitions of the attention kernels: parameters, status word,
// work-unit decoding for padded and packed (varlen) batches.
#pragma once

#include <cstdint>
#include <cuda.h>

#include "sm100_ptx.cuh"

namespace fa {

// Status codes mirrored from include/fa_b200.h (device-side error word).
constexpr int kStatusOk = 0;
constexpr int kStatusTimeout = 4;

// Error word layout: low byte = status code, bits 8..15 = site id of the wait
// that gave up, bits 16..31 = CTA index (saturated).
__device__ __forceinline__ void report_error(int* status, int code, int site) {
  int v = code | ((site & 0xff) << 8) | ((min((int)blockIdx.x, 0xffff)) << 16);
  atomicCAS(status, 0, v);
}

// Work decomposition: a unit is a block of (1 << shift) rows of one
// (sequence, head): 256 query rows (two 128-row tiles) in the forward pass,
// one 128-row query tile (dQ kernel) or one 128-key tile (dK/dV kernel) in
// the backward pass. Units are grouped in levels by their tile index inside
// the sequence; `ascending` walks the levels from tile 0 upwards, otherwise
// from the last tile down, so that for causal attention the heaviest units
// come first. Heads vary fastest, so concurrently running units of one GQA
// group share their K/V tiles in L2. With `level_fastest` (padded batches
// whose units all cost the same: dense, non-causal) the levels vary fastest
// instead: the units running at one time then cover a few (sequence, head)
// pairs whole, and their K/V working set stays in L2 however many pairs the
// batch has.
struct SeqSched {
  const int* cu_seqlens;  // varlen: device [nseq+1]; padded: nullptr
  int nseq;               // padded: B
  int N;                  // padded: sequence length; varlen: max_seqlen
  int heads;              // heads the units run over
  int ascending;          // level order (see above)
  int nlevels;            // ceil(N >> shift)
  const int* level_count; // varlen: smem [nlevels], sequences holding > L units
  int shift;              // log2 of the rows of a unit
  int level_fastest;      // padded only: unit u = pair * nlevels + level (see above)
};

struct Unit {
  int tok0;   // first token of the sequence in the packed token dimension
  int n;      // sequence length
  int qb2;    // index of the unit inside its sequence
  int h;      // head
  int seq;    // sequence (batch) index
};

__device__ __forceinline__ Unit decode_unit(const SeqSched& s, int u) {
  Unit r;
  if (s.cu_seqlens == nullptr) {
    const int BH = s.nseq * s.heads;
    const int level = s.level_fastest ? u % s.nlevels : u / BH;
    const int rem = s.level_fastest ? u / s.nlevels : u - level * BH;
    r.qb2 = s.ascending ? level : (s.nlevels - 1 - level);
    r.h = rem % s.heads;
    r.seq = rem / s.heads;
    r.tok0 = r.seq * s.N;
    r.n = s.N;
    return r;
  }
  int L;
  if (s.ascending) {
    for (L = 0; L < s.nlevels - 1; ++L) {
      const int c = s.level_count[L] * s.heads;
      if (u < c) break;
      u -= c;
    }
  } else {
    for (L = s.nlevels - 1; L > 0; --L) {
      const int c = s.level_count[L] * s.heads;
      if (u < c) break;
      u -= c;
    }
  }
  const int rank = u / s.heads;
  r.h = u - rank * s.heads;
  r.qb2 = L;
  const int round_up = (1 << s.shift) - 1;
  int k = 0;
  int prev = __ldg(s.cu_seqlens);
  for (int q = 0; q < s.nseq; ++q) {
    const int nxt = __ldg(s.cu_seqlens + q + 1);
    const int n = nxt - prev;
    if (((n + round_up) >> s.shift) > L) {
      if (k == rank) {
        r.seq = q;
        r.tok0 = prev;
        r.n = n;
        return r;
      }
      ++k;
    }
    prev = nxt;
  }
  r.seq = 0;
  r.tok0 = 0;
  r.n = 0;  // unreachable for consistent inputs; treated as empty
  return r;
}

// Counts, for a varlen batch, the sequences holding more than L units for
// every level L (shared-memory table, all threads of the block take part)
// and returns the total number of units times `heads`.
__device__ __forceinline__ int varlen_level_table(int* level_count, const int* cu, int nseq, int nlevels, int shift,
                                                  int heads, int nthreads) {
  const int tid = threadIdx.x;
  for (int L = tid; L < nlevels; L += nthreads) level_count[L] = 0;
  __syncthreads();
  const int round_up = (1 << shift) - 1;
  for (int s = tid; s < nseq; s += nthreads) {
    const int n = __ldg(cu + s + 1) - __ldg(cu + s);
    const int nl = min((n + round_up) >> shift, nlevels);
    for (int L = 0; L < nl; ++L) atomicAdd(&level_count[L], 1);
  }
  __syncthreads();
  int tot = 0;
  for (int L = 0; L < nlevels; ++L) tot += level_count[L];
  return tot * heads;
}

// Static persistent schedule in snake order: round r visits CTAs forwards when
// r is even and backwards when odd, so with units sorted heaviest first each
// CTA's total work evens out (a cheap approximation of longest-first).
__device__ __forceinline__ int unit_of(int round, int cta, int grid) {
  return round * grid + ((round & 1) ? (grid - 1 - cta) : cta);
}

}  // namespace fa
