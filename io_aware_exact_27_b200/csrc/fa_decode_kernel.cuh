// Decode: a few new query rows per sequence against a long key/value cache
// (the KV-cache entry point of the Dao-AILab repository overview), split
// over the cache ("split-KV") so that small batches still fill the GPU,
// and the per-split results combined through their log-sum-exp.
//
// Query i of Nq sits at position L_b - Nq + i of sequence b (L_b valid
// cache rows); causal attention lets it see keys 0 .. L_b - Nq + i. A row
// that sees no key gets O = 0 and LSE = -inf.
//
// This path reads the whole cache once per step and does 4*R FMAs per cache
// element for R = Nq * (Hq/Hkv) <= 16 query rows: it is bound by HBM
// bandwidth, so it runs on the CUDA cores with the K/V tiles staged in shared
// memory by TMA, instead of padding the rows up to a tensor-core tile.
//
//   fa_decode_kernel  grid (split, kv head, batch), 128 threads:
//     scores  thread = key of the 128-key tile, all R rows
//     softmax warp = row (rows w, w+4, ...), lanes over the 128 keys
//     P V     thread = output column, R fp32 accumulators
//   fa_decode_merge_kernel  one warp per (batch, query, head) row: combines
//     the splits' (O_r, LSE_r): LSE = log sum exp LSE_r, O = sum exp(LSE_r - LSE) O_r.
#pragma once

#include "fa_common.cuh"

namespace fa {

constexpr int kDecThreads = 128;
constexpr int kDecRows = 16;     // max Nq * (Hq/Hkv)
constexpr int kDecKeys = 128;    // keys per tile
constexpr int kDecStages = 2;

struct DecArgs {
  const void* q;              // [B, Nq, Hq, d] bf16
  const int* cache_seqlens;   // [B] device
  void* o;                    // [B, Nq, Hq, d] bf16 (single split)
  float* lse;                 // [B, Hq, Nq] (single split)
  float* part_o;              // [splits][B][Nq][Hq][d] fp32 (several splits)
  float* part_lse;            // [splits][B][Hq][Nq]
  int B, Nq, Hq, Hkv, Ncache;
  int splits, chunk;          // keys per split (multiple of 128)
  int causal;
  float scale_log2;
  uint64_t timeout_ns;
  int* status;
};

template <int D>
struct DecSmem {
  static constexpr int kTileBytes = kDecKeys * D * 2;
  alignas(1024) uint8_t k[kDecStages][kTileBytes];
  alignas(1024) uint8_t v[kDecStages][kTileBytes];
  alignas(16) float q[kDecRows][D];
  alignas(16) float p[kDecRows][kDecKeys];   // scores, then probabilities of a tile
  float m[kDecRows], l[kDecRows], alpha[kDecRows];
  uint64_t full[kDecStages];
  int abort;
};

// Element (row r, column c) of a 128-row tile stored as D/64 TMA boxes of
// 128 rows x 128 bytes with the 128-byte swizzle: byte offset of the
// 16-byte chunk holding columns 8*(c/8) .. +7.
__device__ __forceinline__ int sw128_chunk(int r, int c) {
  return (c >> 6) * 16384 + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4);
}

template <int D>
__global__ void __launch_bounds__(kDecThreads)
    fa_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const DecArgs a) {
  using Smem = DecSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int G = a.Hq / a.Hkv;
  const int R = a.Nq * G;  // rows r = i*G + g  ->  query i, head hk*G + g
  const int Lb = min(max(__ldg(a.cache_seqlens + b), 0), a.Ncache);
  const int k_begin = split * a.chunk;
  const int k_end = min(Lb, k_begin + a.chunk);
  const int ntiles = k_end > k_begin ? (k_end - k_begin + kDecKeys - 1) / kDecKeys : 0;
  const float cl = a.scale_log2;

  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) mbar_init(smem_u32(&sm.full[s]), 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  // query rows as fp32
  for (int e = tid; e < R * D; e += kDecThreads) {
    const int r = e / D, c = e - r * D;
    const int i = r / G, g = r - i * G;
    const __nv_bfloat16* qp = reinterpret_cast<const __nv_bfloat16*>(a.q) +
                              ((static_cast<size_t>(b) * a.Nq + i) * a.Hq + hk * G + g) * D + c;
    sm.q[r][c] = __bfloat162float(*qp);
  }
  if (tid < kDecRows) {
    sm.m[tid] = -INFINITY;
    sm.l[tid] = 0.f;
  }
  __syncthreads();
  const int row0 = b * a.Ncache + k_begin;  // first cache token of this split
  if (tid == 0) {
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    for (int t = 0; t < min(ntiles, kDecStages); ++t) {
      const uint32_t bar = smem_u32(&sm.full[t]);
      mbar_expect_tx(bar, 2 * Smem::kTileBytes);
#pragma unroll
      for (int bx = 0; bx < D / 64; ++bx) {
        tma_load_3d(smem_u32(sm.k[t]) + bx * 16384, &tm_k, bar, bx * 64, hk, row0 + t * kDecKeys);
        tma_load_3d(smem_u32(sm.v[t]) + bx * 16384, &tm_v, bar, bx * 64, hk, row0 + t * kDecKeys);
      }
    }
  }
  // P V: thread owns output column c, rows rg, rg + CPT, ...
  constexpr int CPT = 128 / D;  // thread groups over the rows
  const int col = tid % D, rg = tid / D;
  float o[kDecRows / CPT];
#pragma unroll
  for (int x = 0; x < kDecRows / CPT; ++x) o[x] = 0.f;

  bool ok = true;
  int issued = min(ntiles, kDecStages);
  for (int t = 0; t < ntiles; ++t) {
    const int st = t % kDecStages;
    ok = __syncthreads_and(mbar_wait(smem_u32(&sm.full[st]), (t / kDecStages) & 1, &sm.abort, a.timeout_ns));
    if (!ok) {
      if (tid == 0) report_error(a.status, kStatusTimeout, 90);
      break;
    }
    const int kbase = k_begin + t * kDecKeys;
    // ---- scores: thread = key
    {
      const int kk = tid;
      const int key = kbase + kk;
      float acc[kDecRows];
#pragma unroll
      for (int r = 0; r < kDecRows; ++r) acc[r] = 0.f;
#pragma unroll 4
      for (int cc = 0; cc < D / 8; ++cc) {
        const uint4 kv = *reinterpret_cast<const uint4*>(sm.k[st] + sw128_chunk(kk, cc * 8));
        const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kv);
        float kf[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(k2[e]);
          kf[2 * e] = f.x;
          kf[2 * e + 1] = f.y;
        }
#pragma unroll
        for (int r = 0; r < kDecRows; ++r) {
          if (r < R) {
            const float4 q0 = *reinterpret_cast<const float4*>(&sm.q[r][cc * 8]);
            const float4 q1 = *reinterpret_cast<const float4*>(&sm.q[r][cc * 8 + 4]);
            acc[r] = fmaf(q0.x, kf[0], acc[r]);
            acc[r] = fmaf(q0.y, kf[1], acc[r]);
            acc[r] = fmaf(q0.z, kf[2], acc[r]);
            acc[r] = fmaf(q0.w, kf[3], acc[r]);
            acc[r] = fmaf(q1.x, kf[4], acc[r]);
            acc[r] = fmaf(q1.y, kf[5], acc[r]);
            acc[r] = fmaf(q1.z, kf[6], acc[r]);
            acc[r] = fmaf(q1.w, kf[7], acc[r]);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < kDecRows; ++r) {
        if (r < R) {
          const int i = r / G;
          const bool vis = key < k_end && !(a.causal && key > Lb - a.Nq + i);
          sm.p[r][kk] = vis ? acc[r] * cl : -INFINITY;
        }
      }
    }
    __syncthreads();
    // ---- online softmax: warp per row, 4 keys per lane
    for (int r = warp; r < R; r += 4) {
      float sv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) sv[u] = sm.p[r][lane + 32 * u];
      float mx = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_old = sm.m[r];
      const float m_new = fmaxf(m_old, mx);
      float alpha = 1.f, sum = 0.f;
      if (m_new != -INFINITY) {
        alpha = ex2_approx(m_old - m_new);  // 0 while m_old is -inf
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float p = ex2_approx(sv[u] - m_new);
          sm.p[r][lane + 32 * u] = p;
          sum += p;
        }
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) sm.p[r][lane + 32 * u] = 0.f;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      if (lane == 0) {
        sm.l[r] = sm.l[r] * alpha + sum;
        sm.m[r] = m_new;
        sm.alpha[r] = alpha;
      }
    }
    __syncthreads();
    // ---- O += P V: thread = output column
    {
#pragma unroll
      for (int x = 0; x < kDecRows / CPT; ++x) {
        const int r = rg + CPT * x;
        if (r < R) o[x] *= sm.alpha[r];
      }
      const uint8_t* vt = sm.v[st];
#pragma unroll 2
      for (int k4 = 0; k4 < kDecKeys; k4 += 4) {
        float vv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int kk = k4 + u;
          const __nv_bfloat16* vp =
              reinterpret_cast<const __nv_bfloat16*>(vt + sw128_chunk(kk, col)) + (col & 7);
          vv[u] = __bfloat162float(*vp);
        }
#pragma unroll
        for (int x = 0; x < kDecRows / CPT; ++x) {
          const int r = rg + CPT * x;
          if (r < R) {
            const float4 p4 = *reinterpret_cast<const float4*>(&sm.p[r][k4]);
            o[x] = fmaf(p4.x, vv[0], o[x]);
            o[x] = fmaf(p4.y, vv[1], o[x]);
            o[x] = fmaf(p4.z, vv[2], o[x]);
            o[x] = fmaf(p4.w, vv[3], o[x]);
          }
        }
      }
    }
    __syncthreads();  // tile st and the probabilities are free again
    if (tid == 0 && issued < ntiles) {
      const uint32_t bar = smem_u32(&sm.full[st]);
      mbar_expect_tx(bar, 2 * Smem::kTileBytes);
#pragma unroll
      for (int bx = 0; bx < D / 64; ++bx) {
        tma_load_3d(smem_u32(sm.k[st]) + bx * 16384, &tm_k, bar, bx * 64, hk, row0 + issued * kDecKeys);
        tma_load_3d(smem_u32(sm.v[st]) + bx * 16384, &tm_v, bar, bx * 64, hk, row0 + issued * kDecKeys);
      }
      ++issued;
    }
  }
  if (!ok) {
    // let issued loads land before the CTA exits
    if (tid == 0)
      for (int t = max(0, issued - kDecStages); t < issued; ++t)
        mbar_wait(smem_u32(&sm.full[t % kDecStages]), (t / kDecStages) & 1, nullptr, a.timeout_ns);
    __syncthreads();
    return;
  }
  // ---- results of this split
#pragma unroll
  for (int x = 0; x < kDecRows / CPT; ++x) {
    const int r = rg + CPT * x;
    if (r >= R) continue;
    const int i = r / G, g = r - i * G, hq = hk * G + g;
    const float l = sm.l[r];
    const float val = l > 0.f ? o[x] / l : 0.f;
    const float lse = l > 0.f ? sm.m[r] * 0.6931471805599453f + logf(l) : -INFINITY;
    const size_t orow = (static_cast<size_t>(b) * a.Nq + i) * a.Hq + hq;
    if (a.splits == 1) {
      reinterpret_cast<__nv_bfloat16*>(a.o)[orow * D + col] = __float2bfloat16_rn(val);
      if (col == 0) a.lse[(static_cast<size_t>(b) * a.Hq + hq) * a.Nq + i] = lse;
    } else {
      const size_t ps = static_cast<size_t>(split) * a.B * a.Nq * a.Hq;
      a.part_o[(ps + orow) * D + col] = val;
      if (col == 0) a.part_lse[ps + (static_cast<size_t>(b) * a.Hq + hq) * a.Nq + i] = lse;
    }
  }
}

// One warp per (batch, query, head) row.
template <int D>
__global__ void __launch_bounds__(256) fa_decode_merge_kernel(const DecArgs a) {
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(a.B) * a.Nq * a.Hq;
  const long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (w >= rows) return;
  const int hq = static_cast<int>(w % a.Hq);
  const int i = static_cast<int>((w / a.Hq) % a.Nq);
  const int b = static_cast<int>(w / (static_cast<long long>(a.Hq) * a.Nq));
  const size_t per_split = static_cast<size_t>(a.B) * a.Nq * a.Hq;
  const size_t li = (static_cast<size_t>(b) * a.Hq + hq) * a.Nq + i;
  float m = -INFINITY;
  for (int r = 0; r < a.splits; ++r) m = fmaxf(m, a.part_lse[r * per_split + li]);
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float lse = -INFINITY;
  if (m != -INFINITY) {
    float s = 0.f;
    for (int r = 0; r < a.splits; ++r) s += expf(a.part_lse[r * per_split + li] - m);
    lse = m + logf(s);
    for (int r = 0; r < a.splits; ++r) {
      const float wgt = expf(a.part_lse[r * per_split + li] - lse);
      const float* po = a.part_o + (r * per_split + static_cast<size_t>(w)) * D;
#pragma unroll
      for (int e = 0; e < PER; ++e) acc[e] = fmaf(wgt, po[lane + 32 * e], acc[e]);
    }
  }
  __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.o) + static_cast<size_t>(w) * D;
#pragma unroll
  for (int e = 0; e < PER; ++e) orow[lane + 32 * e] = __float2bfloat16_rn(acc[e]);
  if (lane == 0) a.lse[li] = lse;
}

}  // namespace fa
