// Merge of attention partials over disjoint key sets (context-parallel ring
// attention across GPUs, the multi-GPU variants of the topic page "Flash
// Attention and Efficient Transformer Mechanisms"): each partial (O_t, LSE_t)
// is exact attention over one key shard, normalised by its own sum; over all
// shards
//   LSE = log sum_t exp LSE_t,   O = sum_t exp(LSE_t - LSE) O_t
// (the LSE merge of key partitions). The partials are bf16 O and fp32 LSE as
// the forward kernel writes them; the sums run in fp32.
#pragma once

#include "fa_common.cuh"

namespace fa {

struct MergeArgs {
  const void* o_parts;     // [nparts][rows, d] bf16, rows = (b, n, h)
  const float* lse_parts;  // [nparts][B, H, N]
  void* o;                 // [rows, d] bf16
  float* lse;              // [B, H, N]
  long long rows;          // B * N * H
  int N, H, nparts;
};

// D/8 lanes per (batch, token, head) row (16-byte loads, 8 columns per lane),
// 32/(D/8) rows per warp. The lanes of a row stride over the partials for the
// maximum and the sum of exp(LSE_t - max); then each lane accumulates its 8
// columns over the partials in order, the loads of kMergeBatch partials
// issued before their sums.
constexpr int kMergeBatch = 4;
template <int D>
__global__ void __launch_bounds__(256) fa_merge_kernel(const MergeArgs a) {
  constexpr int LPR = D / 8;  // lanes per row
  const int lane = threadIdx.x & 31;
  const int sl = lane % LPR;
  const long long w = ((static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5) * (32 / LPR) + lane / LPR;
  const bool live = w < a.rows;
  const long long wr = live ? w : a.rows - 1;  // finished rows still join the shuffles
  const int h = static_cast<int>(wr % a.H);
  const long long bn = wr / a.H;  // b * N + n
  const int n = static_cast<int>(bn % a.N);
  const long long b = bn / a.N;
  const size_t li = (static_cast<size_t>(b) * a.H + h) * a.N + n;
  const size_t lstride = static_cast<size_t>(a.rows);  // one partial's LSE entries (B*H*N)
  float m = -INFINITY;
  for (int t = sl; t < a.nparts; t += LPR) m = fmaxf(m, a.lse_parts[t * lstride + li]);
#pragma unroll
  for (int off = LPR / 2; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float sum = 0.f;
  if (m != -INFINITY)
    for (int t = sl; t < a.nparts; t += LPR) sum += expf(a.lse_parts[t * lstride + li] - m);
#pragma unroll
  for (int off = LPR / 2; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const float lse = m != -INFINITY ? m + logf(sum) : -INFINITY;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  if (lse != -INFINITY) {
    const __nv_bfloat16* base = reinterpret_cast<const __nv_bfloat16*>(a.o_parts) + static_cast<size_t>(wr) * D + sl * 8;
    for (int t0 = 0; t0 < a.nparts; t0 += kMergeBatch) {
      uint4 pv[kMergeBatch];
      float wgt[kMergeBatch];
#pragma unroll
      for (int u = 0; u < kMergeBatch; ++u) {
        const int t = t0 + u;
        wgt[u] = 0.f;
        if (t < a.nparts) {
          pv[u] = __ldg(reinterpret_cast<const uint4*>(base + t * lstride * D));
          wgt[u] = expf(a.lse_parts[t * lstride + li] - lse);  // 0 for a partial that saw no key
        }
      }
#pragma unroll
      for (int u = 0; u < kMergeBatch; ++u) {
        if (t0 + u >= a.nparts) break;
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&pv[u]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(p2[e]);
          acc[2 * e] = fmaf(wgt[u], f.x, acc[2 * e]);
          acc[2 * e + 1] = fmaf(wgt[u], f.y, acc[2 * e + 1]);
        }
      }
    }
  }
  if (live) {
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.o) + static_cast<size_t>(w) * D + sl * 8;
    *reinterpret_cast<uint4*>(out) = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                                pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
    if (sl == 0) a.lse[li] = lse;
  }
}

// Sum of gradient partials over key blocks (ring attention backward): acc
// (fp32) = part, or acc + part, 8 elements per thread (16-byte bf16 loads);
// with `out`, also bf16(acc). part may be null (only the conversion).
struct AccArgs {
  float* acc;
  const void* part;  // bf16 or null
  void* out;         // bf16 or null
  long long n8;      // count / 8
  int first;
};

__global__ void __launch_bounds__(256) fa_grad_accumulate_kernel(const AccArgs a) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= a.n8) return;
  float4* accp = reinterpret_cast<float4*>(a.acc) + 2 * i;
  float v[8];
  if (a.first) {
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = 0.f;
  } else {
    const float4 x0 = accp[0], x1 = accp[1];
    v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w;
    v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
  }
  if (a.part != nullptr) {
    const uint4 p = __ldg(reinterpret_cast<const uint4*>(a.part) + i);
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&p);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(p2[e]);
      v[2 * e] += f.x;
      v[2 * e + 1] += f.y;
    }
  }
  accp[0] = make_float4(v[0], v[1], v[2], v[3]);
  accp[1] = make_float4(v[4], v[5], v[6], v[7]);
  if (a.out != nullptr)
    reinterpret_cast<uint4*>(a.out)[i] =
        make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}

}  // namespace fa
