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

// Work decomposition of the forward pass: a unit is 256 query rows (two
// 128-row tiles) of one (sequence, query head). Units are ordered heaviest
// first for causal attention (more key blocks to visit), and query heads vary
// fastest so that concurrently running units of one GQA group share their
// K/V tiles in L2.
struct SeqSched {
  const int* cu_seqlens;  // varlen: device [nseq+1]; padded: nullptr
  int nseq;               // padded: B
  int N;                  // padded: sequence length; varlen: max_seqlen
  int Hq;
  int causal;
  int nlevels;            // number of 256-row levels (ceil(N / 256))
  const int* level_count; // varlen: smem [nlevels], sequences with > L units
};

struct Unit {
  int tok0;   // first token of the sequence in the packed token dimension
  int n;      // sequence length
  int qb2;    // index of the 256-row block inside the sequence
  int h;      // query head
  int seq;    // sequence (batch) index
};

__device__ __forceinline__ Unit decode_unit(const SeqSched& s, int u) {
  Unit r;
  if (s.cu_seqlens == nullptr) {
    const int BH = s.nseq * s.Hq;
    const int level = u / BH;
    const int rem = u - level * BH;
    r.qb2 = s.causal ? (s.nlevels - 1 - level) : level;
    r.h = rem % s.Hq;
    r.seq = rem / s.Hq;
    r.tok0 = r.seq * s.N;
    r.n = s.N;
    return r;
  }
  // varlen: walk levels from the top; level L holds the units with qb2 == L
  int L = s.nlevels - 1;
  for (; L > 0; --L) {
    const int c = s.level_count[L] * s.Hq;
    if (u < c) break;
    u -= c;
  }
  const int rank = u / s.Hq;
  r.h = u - rank * s.Hq;
  r.qb2 = L;
  // the rank-th sequence holding more than L units
  int k = 0;
  int prev = __ldg(s.cu_seqlens);
  for (int q = 0; q < s.nseq; ++q) {
    const int nxt = __ldg(s.cu_seqlens + q + 1);
    const int n = nxt - prev;
    if (((n + 255) >> 8) > L) {
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

}  // namespace fa
