// Block-scaled e4m3 inputs for the fp8 forward, with optional incoherent
// processing: the rows of Q and K are first rotated by the orthogonal
// Hadamard matrix H_d / sqrt(d) (FA-3 summary, contribution 3: FP8 with lower
// error than per-tensor quantisation; the technique is not named there, the
// rotation is the reading taken). (Q H)(K H)^T = Q K^T, so the scores are
// unchanged; an outlier channel is spread over all d channels before the
// rounding.
//
// One CTA per (batch, head, 128-row block), 8 warps x 16 rows, one row per
// warp-instruction (D/32 elements per lane):
//   1. load the bf16 row as fp32; with rotation, the fast Walsh-Hadamard
//      transform: stage widths h = 1, 2, ..., D/2, each pair (j, j+h) with bit
//      h of j clear becomes (x_j + x_{j+h}, x_j - x_{j+h}); widths below
//      D/32 inside a lane, the rest between lanes (shuffle with lane ^ h/(D/32));
//      then one fp32 multiply by fp32(1/sqrt(D));
//   2. amax over the block; s = amax / 448 (1 for an all-zero block);
//   3. codes = round-to-nearest-even e4m3 of the fp32 quotient y / s.
// Every step is a single IEEE fp32 operation in a fixed order, so the codes
// and scales are bit-identical to the same steps done in float32 anywhere.
#pragma once

#include <type_traits>

#include "fa_common.cuh"

namespace fa {

struct QuantArgs {
  const void* x;   // [B, N, H, D] bf16
  uint8_t* codes;  // [B, N, H, D] e4m3
  float* scales;   // [B, H, nblk]
  int B, N, H, nblk;
  int rotate;
  float rscale;    // fp32(1/sqrt(D))
};

template <int D>
__global__ void __launch_bounds__(256) fa_quant_kernel(const QuantArgs a) {
  constexpr int E = D / 32;  // elements per lane
  constexpr int RPW = 16;    // rows per warp
  __shared__ float wmax[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int n_first = blk * 128 + warp * RPW;
  // the warp's 16 rows are loaded first (all loads in flight together), then
  // converted and rotated one by one
  using Raw = typename std::conditional<E == 4, uint2, uint32_t>::type;
  Raw raw[RPW];
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    const int n = n_first + r;
    if (n < a.N)
      raw[r] = __ldg(reinterpret_cast<const Raw*>(reinterpret_cast<const __nv_bfloat16*>(a.x) +
                                                  ((static_cast<size_t>(b) * a.N + n) * a.H + h) * D + lane * E));
    else
      raw[r] = Raw{};
  }
  float y[RPW][E];
  float amax = 0.f;
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    float v[E];
    if constexpr (E == 4) {
      const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[r].x));
      const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[r].y));
      v[0] = f0.x;
      v[1] = f0.y;
      v[2] = f1.x;
      v[3] = f1.y;
    } else {
      const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[r]));
      v[0] = f0.x;
      v[1] = f0.y;
    }
    if (a.rotate) {  // uniform over the grid
      // widths inside the lane (element j = lane*E + e)
#pragma unroll
      for (int w = 1; w < E; w *= 2) {
        float t[E];
#pragma unroll
        for (int e = 0; e < E; ++e) t[e] = (e & w) ? v[e - w] - v[e] : v[e] + v[e + w];
#pragma unroll
        for (int e = 0; e < E; ++e) v[e] = t[e];
      }
      // widths between lanes: bit w of j is bit w/E of the lane
#pragma unroll
      for (int lw = 1; lw < 32; lw *= 2) {
        const bool upper = lane & lw;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const float p = __shfl_xor_sync(0xffffffffu, v[e], lw);
          v[e] = upper ? p - v[e] : v[e] + p;
        }
      }
#pragma unroll
      for (int e = 0; e < E; ++e) v[e] = v[e] * a.rscale;
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
      y[r][e] = v[e];
      amax = fmaxf(amax, fabsf(v[e]));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if (lane == 0) wmax[warp] = amax;
  __syncthreads();
  float m = wmax[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) m = fmaxf(m, wmax[w]);
  const float s = m > 0.f ? m / 448.f : 1.f;
  if (threadIdx.x == 0) a.scales[(static_cast<size_t>(b) * a.H + h) * a.nblk + blk] = s;
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    const int n = n_first + r;
    if (n >= a.N) break;
    uint8_t* dst = a.codes + ((static_cast<size_t>(b) * a.N + n) * a.H + h) * D + lane * E;
    if constexpr (E == 4) {
      *reinterpret_cast<uint32_t*>(dst) = pack_e4m3x4(y[r][0] / s, y[r][1] / s, y[r][2] / s, y[r][3] / s);
    } else {
      uint16_t c;
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c) : "f"(y[r][1] / s), "f"(y[r][0] / s));
      *reinterpret_cast<uint16_t*>(dst) = c;
    }
  }
}

// The inverse map, input of the fp8 backward: bf16 values in the original
// space from the codes and scales. One CTA per (batch, head, 128-row block),
// 8 warps x 16 rows; per element, each step one IEEE fp32 operation in a
// fixed order: code (exact e4m3 -> f16 -> f32) times the block's scale; with
// `unrotate` the same butterflies and 1/sqrt(D) multiply as the quantiser
// (H_D / sqrt(D) is its own inverse); round to nearest even bf16.
struct DequantArgs {
  const uint8_t* codes;  // [B, N, H, D] e4m3
  const float* scales;   // [B, H, nblk]
  void* x;               // [B, N, H, D] bf16 (out)
  int B, N, H, nblk;
  int unrotate;
  float rscale;          // fp32(1/sqrt(D))
};

template <int D>
__global__ void __launch_bounds__(256) fa_dequant_kernel(const DequantArgs a) {
  constexpr int E = D / 32;  // elements per lane
  constexpr int RPW = 16;    // rows per warp
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const float s = a.scales[(static_cast<size_t>(b) * a.H + h) * a.nblk + blk];
#pragma unroll 4
  for (int r = 0; r < RPW; ++r) {
    const int n = blk * 128 + warp * RPW + r;  // uniform over the warp
    if (n >= a.N) break;
    const size_t off = ((static_cast<size_t>(b) * a.N + n) * a.H + h) * D + lane * E;
    float v[E];
    if constexpr (E == 4) {
      const uint32_t c = __ldg(reinterpret_cast<const uint32_t*>(a.codes + off));
      const uint32_t lo = e4m3x2_to_f16x2(static_cast<uint16_t>(c & 0xffffu));
      const uint32_t hi = e4m3x2_to_f16x2(static_cast<uint16_t>(c >> 16));
      const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&lo));
      const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&hi));
      v[0] = f0.x * s;
      v[1] = f0.y * s;
      v[2] = f1.x * s;
      v[3] = f1.y * s;
    } else {
      const uint16_t c = __ldg(reinterpret_cast<const uint16_t*>(a.codes + off));
      const uint32_t w = e4m3x2_to_f16x2(c);
      const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&w));
      v[0] = f0.x * s;
      v[1] = f0.y * s;
    }
    if (a.unrotate) {  // uniform over the grid
#pragma unroll
      for (int w = 1; w < E; w *= 2) {
        float t[E];
#pragma unroll
        for (int e = 0; e < E; ++e) t[e] = (e & w) ? v[e - w] - v[e] : v[e] + v[e + w];
#pragma unroll
        for (int e = 0; e < E; ++e) v[e] = t[e];
      }
#pragma unroll
      for (int lw = 1; lw < 32; lw *= 2) {
        const bool upper = lane & lw;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const float p = __shfl_xor_sync(0xffffffffu, v[e], lw);
          v[e] = upper ? p - v[e] : v[e] + p;
        }
      }
#pragma unroll
      for (int e = 0; e < E; ++e) v[e] = v[e] * a.rscale;
    }
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.x) + off;
    if constexpr (E == 4)
      *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
    else
      *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(v[0], v[1]);
  }
}

}  // namespace fa
