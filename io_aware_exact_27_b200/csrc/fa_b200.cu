// C-ABI of the attention library: argument validation, TMA tensor-map
// encoding, launch configuration and the device status word. The kernels
// live in the fa_*_kernel.cuh headers included below (one translation unit).
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/fa_b200.h"
#include "fa_bwd_kernel.cuh"
#include "fa_bwd_pre_kernel.cuh"
#include "fa_fwd_kernel.cuh"
#include "fa_decode_kernel.cuh"
#include "fa_merge_kernel.cuh"
#include "fa_quant_kernel.cuh"

namespace {

__device__ int g_status_word;  // first device-side error since the last fa_get_status()

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::atomic<uint64_t> g_timeout_ns{4000000000ull};
std::atomic<int> g_inject{0};
std::atomic<int> g_last_word{0};

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;
  int sms = 0;
  int cc = 0;
  int* status = nullptr;     // device address of g_status_word
  bool fwd_attr[3][2] = {};  // [bf16 d64, bf16 d128, fp8][block-sparse]
  bool bwd_attr[2][3] = {};  // [d == 128][bf16 dense, block-sparse, fp8 scores]
  bool dec_attr[2] = {false, false};
  // the backward runs its dQ kernel beside the dK/dV kernel: a second stream
  // and two events, created on first use
  cudaStream_t side = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
DeviceState g_dev[kMaxDevices];
std::mutex g_mu;

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// Per-device facts, looked up once per device with that device current.
fa_status_t device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& s = g_dev[dev];
  if (!s.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return FA_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return FA_ERR_CUDA;
    s.cc = major * 10 + minor;
    s.sms = sms;
    s.status = static_cast<int*>(p);
    s.ready = true;
  }
  if (s.cc != 100) return FA_ERR_UNSUPPORTED;
  *out = &s;
  return FA_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// [tokens, heads, d] tensor with 128-row x 64-element (128-byte) boxes, 128B swizzle.
fa_status_t encode_rows(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, int tokens,
                        int heads, int d, CUtensorMapL2promotion promo = CU_TENSOR_MAP_L2_PROMOTION_L2_256B) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return FA_ERR_CUDA;
  const int box_inner = 128 / elem_bytes;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads),
                        static_cast<cuuint64_t>(tokens)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * elem_bytes,
                           static_cast<cuuint64_t>(heads) * d * elem_bytes};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), 1, 128};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

fa_status_t check_common(const void* q, const void* k, const void* v, const void* o, const float* lse, int Hq,
                         int Hkv, int d, float scale) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return FA_ERR_INVALID_ARG;
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

template <int D, bool F8 = false, bool SPARSE = false>
fa_status_t launch_fwd(DeviceState* ds, const void* q, const void* k, const void* v, fa::FwdArgs a, int tokens,
                       long long units_bound, cudaStream_t stream) {
  constexpr int STAGES = F8 ? 6 : 4;
  using Smem = fa::FwdSmem<D, STAGES, F8>;
  auto kern = fa::fa_fwd_sm100_kernel<D, STAGES, F8, SPARSE>;
  const int smem = static_cast<int>(sizeof(Smem)) + 1024;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    bool& done = ds->fwd_attr[F8 ? 2 : (D == 128 ? 1 : 0)][SPARSE ? 1 : 0];
    if (!done) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return FA_ERR_CUDA;
      done = true;
    }
  }
  CUtensorMap tq, tk, tv;
  fa_status_t st;
  const CUtensorMapDataType dt = F8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  constexpr int EB = F8 ? 1 : 2;
  if ((st = encode_rows(&tq, q, dt, EB, tokens, a.Hq, D)) != FA_OK) return st;
  if ((st = encode_rows(&tk, k, dt, EB, tokens, a.Hkv, D)) != FA_OK) return st;
  if ((st = encode_rows(&tv, v, dt, EB, tokens, a.Hkv, D)) != FA_OK) return st;
  a.timeout_ns = g_timeout_ns.load();
  a.inject = g_inject.load();
  a.status = ds->status;
  const int grid = static_cast<int>(units_bound < ds->sms ? units_bound : ds->sms);
  if (grid <= 0) return FA_OK;
  kern<<<grid, F8 ? fa::kThreadsFwdF8 : fa::kThreadsFwd, smem, stream>>>(tq, tk, tv, a);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status_t fwd_dispatch(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu, int nseq,
                         int N, int total_T, int Hq, int Hkv, int d, int causal, float scale, void* stream,
                         const uint8_t* block_mask = nullptr) {
  fa_status_t st = check_common(q, k, v, o, lse, Hq, Hkv, d, scale);
  if (st != FA_OK) return st;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  if ((st = device_state(&ds)) != FA_OK) return st;
  fa::FwdArgs a{};
  a.o = o;
  a.lse = lse;
  a.cu_seqlens = cu;
  a.nseq = nseq;
  a.N = N;
  a.total_T = total_T;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.causal = causal;
  a.scale = scale;
  a.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  a.block_mask = block_mask;
  a.nqb = (N + fa::kBM - 1) / fa::kBM;
  const long long nlev = (N + 255) / 256;
  long long bound;
  if (cu == nullptr) {
    a.lse_head_stride = N;
    bound = static_cast<long long>(nseq) * Hq * nlev;
    a.num_units = static_cast<int>(bound);
  } else {
    a.lse_head_stride = total_T;
    const long long by_len = static_cast<long long>(nseq) * nlev;
    const long long by_tok = (static_cast<long long>(total_T) + 255) / 256 + nseq;
    bound = static_cast<long long>(Hq) * (by_len < by_tok ? by_len : by_tok);
    a.num_units = static_cast<int>(bound);  // recomputed exactly on the device
  }
  if (bound > INT32_MAX) return FA_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (block_mask != nullptr)
    return d == 128 ? launch_fwd<128, false, true>(ds, q, k, v, a, total_T, bound, s)
                    : launch_fwd<64, false, true>(ds, q, k, v, a, total_T, bound, s);
  return d == 128 ? launch_fwd<128>(ds, q, k, v, a, total_T, bound, s)
                  : launch_fwd<64>(ds, q, k, v, a, total_T, bound, s);
}

// Floats per head of each backward workspace vector (see fa::ws_offset).
size_t vec_stride(int tokens, int nseq) {
  return ((static_cast<size_t>(tokens) + 3) & ~size_t(3)) + 4 * static_cast<size_t>(nseq) + fa::kVecSlack;
}
size_t vec_bytes(int tokens, int nseq, int Hq) {
  const size_t b = static_cast<size_t>(Hq) * vec_stride(tokens, nseq) * sizeof(float);
  return (b + 255) & ~size_t(255);
}

// Block-sparse backward: the dK/dV work plan and the split units' partial
// sums follow the two workspace vectors. units = B * Hkv * ceil(N/128);
// partial slots: 4 per SM (the plan leaves units unsplit beyond that).
struct SparsePlanLayout {
  long long units, max_slots, max_items, max_steps, rows;
  size_t plan_off, nbuf_off, sbase_off, steps_off, rows_n_off, rows_base_off, rows_list_off, part_off, total;
};
SparsePlanLayout sparse_plan_layout(size_t base, int B, int Hq, int Hkv, int N, int d, int sms) {
  SparsePlanLayout L{};
  const long long nqb = (N + 127) / 128;
  L.units = static_cast<long long>(B) * Hkv * nqb;
  L.max_steps = L.units * (Hq / Hkv) * nqb;  // every (query head, query tile) of every unit
  L.max_slots = 4LL * sms;
  L.max_items = L.units + L.max_slots;
  const size_t plan_ints = 4 + 4 * static_cast<size_t>(L.max_items) + 4 * static_cast<size_t>(L.max_slots);
  L.plan_off = (base + 255) & ~size_t(255);
  L.nbuf_off = (L.plan_off + plan_ints * sizeof(int) + 255) & ~size_t(255);
  L.sbase_off = (L.nbuf_off + static_cast<size_t>(L.units) * sizeof(int) + 255) & ~size_t(255);
  L.steps_off = (L.sbase_off + static_cast<size_t>(L.units) * sizeof(int) + 255) & ~size_t(255);
  // dQ rows: per (query head, query tile) the visible key blocks
  L.rows = static_cast<long long>(Hq) * nqb;
  L.rows_n_off = (L.steps_off + static_cast<size_t>(L.max_steps) * sizeof(int) + 255) & ~size_t(255);
  L.rows_base_off = (L.rows_n_off + static_cast<size_t>(L.rows) * sizeof(int) + 255) & ~size_t(255);
  L.rows_list_off = (L.rows_base_off + static_cast<size_t>(L.rows) * sizeof(int) + 255) & ~size_t(255);
  L.part_off = (L.rows_list_off + static_cast<size_t>(L.rows) * nqb * sizeof(int) + 255) & ~size_t(255);
  L.total = L.part_off + static_cast<size_t>(L.max_slots) * 2 * 128 * d * sizeof(float);
  return L;
}

// F8: the score products S = Q K^T (dQ kernel) and S^T = K Q^T (dK/dV
// kernel) run on the e4m3 codes q8, k8 (block scales in `a`); q, k, v are
// then the bf16 values of the other products.
template <int D, bool SPARSE = false, bool F8 = false>
fa_status_t launch_bwd(DeviceState* ds, const void* q, const void* k, const void* v, const void* dout,
                       fa::BwdArgs a, long long units_dq, long long units_dkdv, int parts, cudaStream_t stream,
                       const void* q8 = nullptr, const void* k8 = nullptr) {
  constexpr int STAGES = 4;
  auto kdq = fa::fa_bwd_dq_kernel<D, STAGES, SPARSE, F8>;
  auto kdkv = fa::fa_bwd_dkdv_kernel<D, STAGES, SPARSE, F8>;
  const int smem_dq = static_cast<int>(sizeof(fa::DqSmem<D, STAGES, F8>)) + 1024;
  const int smem_dkv = static_cast<int>(sizeof(fa::DkvSmem<D, STAGES, F8>)) + 1024;
  auto kpre = fa::fa_bwd_pre_kernel<D>;
  const int smem_pre = static_cast<int>(sizeof(fa::PreSmem)) + 128;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    bool& done = ds->bwd_attr[D == 128 ? 1 : 0][F8 ? 2 : (SPARSE ? 1 : 0)];
    if (!done) {
      if (cudaFuncSetAttribute(kdq, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_dq) != cudaSuccess ||
          cudaFuncSetAttribute(kdkv, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_dkv) != cudaSuccess ||
          cudaFuncSetAttribute(kpre, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_pre) != cudaSuccess)
        return FA_ERR_CUDA;
      done = true;
    }
  }
  CUtensorMap tq, tk, tv, tdo;
  fa_status_t st;
  const int T = a.total_T;
  if ((st = encode_rows(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, T, a.Hq, D)) != FA_OK) return st;
  if ((st = encode_rows(&tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, T, a.Hkv, D)) != FA_OK) return st;
  if ((st = encode_rows(&tv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, T, a.Hkv, D)) != FA_OK) return st;
  if ((st = encode_rows(&tdo, dout, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, T, a.Hq, D)) != FA_OK) return st;
  // the e4m3 code tiles of the fp8 score products (unused otherwise)
  CUtensorMap tq8 = tq, tk8 = tk;
  if (F8) {
    if ((st = encode_rows(&tq8, q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, T, a.Hq, D)) != FA_OK) return st;
    if ((st = encode_rows(&tk8, k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, T, a.Hkv, D)) != FA_OK) return st;
  }
  a.timeout_ns = g_timeout_ns.load();
  a.status = ds->status;
  // D and LSE in base 2: one CTA per SM (a ring of 3 x 64 KB of O and dO
  // chunks), at most one per chunk
  const long long entries = static_cast<long long>(a.Hq) * a.total_T;
  const long long chunk_entries = fa::kPreChunk / (D * 2);
  long long pre_blocks = (entries + chunk_entries - 1) / chunk_entries;
  if (pre_blocks > ds->sms) pre_blocks = ds->sms;
  if (pre_blocks < 1) pre_blocks = 1;
  if (parts & FA_BWD_PREPARE) {
    kpre<<<static_cast<int>(pre_blocks), fa::kPreThreads, smem_pre, stream>>>(a);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  fa::BwdArgs akv = a;
  akv.num_units = static_cast<int>(units_dkdv);
  long long work_dkdv = units_dkdv;  // dense: units; block-sparse: an upper bound of the planned items
  if (SPARSE) work_dkdv = a.plan_max_items;
  const int g1 = static_cast<int>(work_dkdv < ds->sms ? work_dkdv : ds->sms);
  // dK/dV on `stream`; block-sparse: the work plan (one CTA) before it and
  // the sums of the split units' partials after it
  auto run_dkdv = [&]() -> bool {
    if (SPARSE) {
      // the per-CTA share counts one CTA per unit at most: units are only
      // split when far longer than the others, never to widen the grid
      const int share_grid = static_cast<int>(units_dkdv < g1 ? units_dkdv : g1);
      fa::fa_bwd_plan_count_kernel<<<static_cast<int>((units_dkdv + 7) / 8), 256, 0, stream>>>(
          a, static_cast<int>(units_dkdv), a.plan_nbuf);
      if (cudaGetLastError() != cudaSuccess) return false;
      fa::fa_bwd_plan_kernel<<<1, fa::kPlanThreads, 0, stream>>>(a, static_cast<int>(units_dkdv), share_grid,
                                                                 a.plan_max_slots, a.plan_nbuf);
      if (cudaGetLastError() != cudaSuccess) return false;
      fa::fa_bwd_plan_steps_kernel<<<static_cast<int>((units_dkdv + 7) / 8), 256, 0, stream>>>(
          a, static_cast<int>(units_dkdv));
      if (cudaGetLastError() != cudaSuccess) return false;
    }
    kdkv<<<g1, fa::kThreadsBwd, smem_dkv, stream>>>(tq, tk, tv, tdo, tq8, tk8, akv);
    if (cudaGetLastError() != cudaSuccess) return false;
    if (SPARSE) {
      fa::fa_bwd_reduce_kernel<D><<<ds->sms, 256, 0, stream>>>(a);
      if (cudaGetLastError() != cudaSuccess) return false;
    }
    return true;
  };
  fa::BwdArgs aq = a;
  aq.num_units = static_cast<int>(units_dq);
  const int g2 = static_cast<int>(units_dq < ds->sms ? units_dq : ds->sms);
  // dQ on stream `st`; block-sparse: the rows' key-block lists before it
  auto run_dq = [&](cudaStream_t st) -> bool {
    if (SPARSE) {
      const int rows = a.Hq * a.nqb;
      fa::fa_bwd_rows_count_kernel<<<(rows + 7) / 8, 256, 0, st>>>(a, rows);
      fa::fa_bwd_rows_scan_kernel<<<1, fa::kPlanThreads, 0, st>>>(a, rows);
      fa::fa_bwd_rows_list_kernel<<<(rows + 7) / 8, 256, 0, st>>>(a, rows);
      if (cudaGetLastError() != cudaSuccess) return false;
    }
    kdq<<<g2, fa::kThreadsBwd, smem_dq, st>>>(tq, tk, tv, tdo, tq8, tk8, aq);
    return cudaGetLastError() == cudaSuccess;
  };
  if ((parts & FA_BWD_DKDV) && (parts & FA_BWD_DQ) && g1 > 0 && g2 > 0) {
    // dK/dV on the caller's stream and dQ on the side stream, both after the
    // preparation: their persistent CTAs have uneven causal work, and dQ's
    // CTAs take the SMs that dK/dV's leave early. The caller's stream waits
    // for both. Each output is still written by one CTA (deterministic).
    std::lock_guard<std::mutex> lk(g_mu);
    if (ds->side == nullptr) {
      if (cudaStreamCreateWithFlags(&ds->side, cudaStreamNonBlocking) != cudaSuccess ||
          cudaEventCreateWithFlags(&ds->fork, cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&ds->join, cudaEventDisableTiming) != cudaSuccess)
        return FA_ERR_CUDA;
    }
    if (cudaEventRecord(ds->fork, stream) != cudaSuccess || cudaStreamWaitEvent(ds->side, ds->fork, 0) != cudaSuccess)
      return FA_ERR_CUDA;
    if (!run_dkdv()) return FA_ERR_CUDA;
    if (!run_dq(ds->side)) return FA_ERR_CUDA;
    if (cudaEventRecord(ds->join, ds->side) != cudaSuccess || cudaStreamWaitEvent(stream, ds->join, 0) != cudaSuccess)
      return FA_ERR_CUDA;
    return FA_OK;
  }
  if (parts & FA_BWD_DKDV) {
    if (g1 > 0 && !run_dkdv()) return FA_ERR_CUDA;
  }
  if (parts & FA_BWD_DQ) {
    if (g2 > 0 && !run_dq(stream)) return FA_ERR_CUDA;
  }
  return FA_OK;
}

fa_status_t bwd_dispatch(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dout, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                         const int* cu, int nseq, int N, int total_T, int Hq, int Hkv, int d, int causal,
                         float scale, void* stream, int parts = FA_BWD_ALL, const uint8_t* block_mask = nullptr,
                         const void* q8 = nullptr, const void* k8 = nullptr, const float* q_scale = nullptr,
                         const float* k_scale = nullptr) {
  fa_status_t st = check_common(q, k, v, o, lse, Hq, Hkv, d, scale);
  if (st != FA_OK) return st;
  if (!dout || !dq || !dk || !dv || !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) ||
      !aligned(dv, 16))
    return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  const size_t vb = vec_bytes(total_T, nseq, Hq);
  if (workspace == nullptr || !aligned(workspace, 256) || ws_bytes < 2 * vb) return FA_ERR_WORKSPACE;
  DeviceState* ds = nullptr;
  if ((st = device_state(&ds)) != FA_OK) return st;
  SparsePlanLayout L{};
  if (block_mask != nullptr) {
    L = sparse_plan_layout(2 * vb, nseq, Hq, Hkv, N, d, ds->sms);
    if (ws_bytes < L.total) return FA_ERR_WORKSPACE;
    if (L.max_items > INT32_MAX / 4 || L.max_steps > INT32_MAX || L.rows * ((N + 127) / 128) > INT32_MAX)
      return FA_ERR_UNSUPPORTED;
  }
  fa::BwdArgs a{};
  a.o = o;
  a.dout = dout;
  a.lse = lse;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.lse2 = static_cast<float*>(workspace);
  a.dvec = reinterpret_cast<float*>(static_cast<char*>(workspace) + vb);
  a.cu_seqlens = cu;
  a.nseq = nseq;
  a.N = N;
  a.total_T = total_T;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.causal = causal;
  a.scale = scale;
  a.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  a.lse_head_stride = cu ? total_T : N;
  if (vec_stride(total_T, nseq) > static_cast<size_t>(INT32_MAX)) return FA_ERR_UNSUPPORTED;
  a.ws_stride = static_cast<int>(vec_stride(total_T, nseq));
  const long long nt = (N + 127) / 128;
  long long udq, ukv;
  if (cu == nullptr) {
    udq = static_cast<long long>(nseq) * Hq * nt;
    ukv = static_cast<long long>(nseq) * Hkv * nt;
  } else {
    const long long by_len = static_cast<long long>(nseq) * nt;
    const long long by_tok = (static_cast<long long>(total_T) + 127) / 128 + nseq;
    const long long t = by_len < by_tok ? by_len : by_tok;
    udq = t * Hq;  // upper bounds; the exact counts are recomputed on the device
    ukv = t * Hkv;
  }
  if (udq > INT32_MAX) return FA_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (parts <= 0 || parts > FA_BWD_ALL) return FA_ERR_INVALID_ARG;
  a.block_mask = block_mask;
  a.nqb = static_cast<int>(nt);
  if (block_mask != nullptr) {
    char* w = static_cast<char*>(workspace);
    a.plan = reinterpret_cast<int*>(w + L.plan_off);
    a.plan_nbuf = reinterpret_cast<int*>(w + L.nbuf_off);
    a.plan_sbase = reinterpret_cast<int*>(w + L.sbase_off);
    a.plan_steps = reinterpret_cast<int*>(w + L.steps_off);
    a.rows_n = reinterpret_cast<int*>(w + L.rows_n_off);
    a.rows_base = reinterpret_cast<int*>(w + L.rows_base_off);
    a.rows_list = reinterpret_cast<int*>(w + L.rows_list_off);
    a.partials = reinterpret_cast<float*>(w + L.part_off);
    a.plan_max_items = static_cast<int>(L.max_items);
    a.plan_max_slots = static_cast<int>(L.max_slots);
  }
  if (q8 != nullptr) {
    // fp8 scores: padded batches, d = 128 (as the fp8 forward)
    a.q_scale = q_scale;
    a.k_scale = k_scale;
    a.nblk_s = static_cast<int>(nt);
    return launch_bwd<128, false, true>(ds, q, k, v, dout, a, udq, ukv, parts, s, q8, k8);
  }
  if (block_mask != nullptr)
    return d == 128 ? launch_bwd<128, true>(ds, q, k, v, dout, a, udq, ukv, parts, s)
                    : launch_bwd<64, true>(ds, q, k, v, dout, a, udq, ukv, parts, s);
  return d == 128 ? launch_bwd<128>(ds, q, k, v, dout, a, udq, ukv, parts, s)
                  : launch_bwd<64>(ds, q, k, v, dout, a, udq, ukv, parts, s);
}

// ---------------------------------------------------------------- no-allocation backward
// Scratch of fa_bwd_noalloc: a fixed array in device memory, created when the
// library is loaded and held by every GPU that loads it until the process
// exits. Host code must not use the symbol itself as an address (on the host
// it only names the array); its device address is looked up per device below.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;
static __device__ __align__(256) unsigned char g_fa_noalloc_scratch[kNoAllocScratchBytes];
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device; looked up once
// per device (with that device current) and cached.
fa_status_t noalloc_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fa_noalloc_scratch) != cudaSuccess || p == nullptr) return FA_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return FA_OK;
}

// ---------------------------------------------------------------- decode (KV cache)
size_t dec_part_floats(int B, int Nq, int Hq, int d, int splits) {
  return static_cast<size_t>(splits) * B * Nq * Hq * (static_cast<size_t>(d) + 1);
}

// Query rows of one (batch, kv head) unit: a box of {64 columns, G heads,
// Nq queries} from q [B*Nq, Hq, d], landing as R = Nq*G rows of 128 bytes
// (row i*G + g) with the 128-byte swizzle.
fa_status_t encode_query_rows(CUtensorMap* m, const void* q, int B, int Nq, int Hq, int G, int d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return FA_ERR_CUDA;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(Hq),
                        static_cast<cuuint64_t>(B) * static_cast<cuuint64_t>(Nq)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(Hq) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(Nq)};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

template <int D>
fa_status_t launch_decode(DeviceState* ds, const void* kc, const void* vc, fa::DecArgs a, cudaStream_t stream) {
  using Smem = fa::DecSmem<D>;
  auto kern = fa::fa_decode_kernel<D>;
  const int smem = static_cast<int>(sizeof(Smem)) + 1024;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    bool& done = ds->dec_attr[D == 128 ? 1 : 0];
    if (!done) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return FA_ERR_CUDA;
      done = true;
    }
  }
  CUtensorMap tq, tk, tv;
  fa_status_t st;
  const int tokens = a.B * a.Ncache;
  if ((st = encode_query_rows(&tq, a.q, a.B, a.Nq, a.Hq, a.Hq / a.Hkv, D)) != FA_OK) return st;
  // a head's cache row is D*2 bytes: promote L2 fills to no more than that,
  // so that a 64-wide head does not drag its neighbour's row in with it
  const CUtensorMapL2promotion promo = D == 128 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_L2_128B;
  if ((st = encode_rows(&tk, kc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, a.Hkv, D, promo)) != FA_OK) return st;
  if ((st = encode_rows(&tv, vc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, a.Hkv, D, promo)) != FA_OK) return st;
  a.timeout_ns = g_timeout_ns.load();
  a.status = ds->status;
  const int grid = a.num_units < ds->sms ? a.num_units : ds->sms;
  kern<<<grid, fa::kDecThreads, smem, stream>>>(tq, tk, tv, a);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  if (a.splits > 1) {
    const long long rows = static_cast<long long>(a.B) * a.Nq * a.Hq;
    fa::fa_decode_merge_kernel<D><<<static_cast<int>((rows + 7) / 8), 256, 0, stream>>>(a);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  return FA_OK;
}

// Keys per split for a requested split count: whole 128-key tiles.
int dec_chunk_keys(int Ncache, int num_splits) {
  const int per = (Ncache + num_splits - 1) / num_splits;
  return (per + fa::kDecKeys - 1) / fa::kDecKeys * fa::kDecKeys;
}

}  // namespace

extern "C" {

fa_status_t fa_fwd_blocksparse(const void* q, const void* k, const void* v, const unsigned char* block_mask, void* o,
                               float* lse, int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                               void* stream) {
  if (B < 0 || N < 0) return FA_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return FA_OK;
  if (block_mask == nullptr) return FA_ERR_INVALID_ARG;
  if (N > 131072) return FA_ERR_UNSUPPORTED;  // the softmax warps hold a mask row in 32 x 32 bits
  return fwd_dispatch(q, k, v, o, lse, nullptr, B, N, B * N, Hq, Hkv, d, causal, scale, stream, block_mask);
}

fa_status_t fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                   int d, int causal, float scale, void* stream) {
  if (B < 0 || N < 0) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * N == 0) return FA_OK;
  if (static_cast<long long>(B) * N > INT32_MAX) return FA_ERR_UNSUPPORTED;
  return fwd_dispatch(q, k, v, o, lse, nullptr, B, N, B * N, Hq, Hkv, d, causal, scale, stream);
}

fa_status_t fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_seqlens,
                          int nseq, int max_seqlen, int total_T, int Hq, int Hkv, int d, int causal, float scale,
                          void* stream) {
  if (nseq < 0 || total_T < 0 || max_seqlen < 0 || cu_seqlens == nullptr || !aligned(cu_seqlens, 4))
    return FA_ERR_INVALID_ARG;
  if (nseq == 0 || total_T == 0 || max_seqlen == 0) return FA_OK;
  if (max_seqlen > 131072) return FA_ERR_UNSUPPORTED;
  return fwd_dispatch(q, k, v, o, lse, cu_seqlens, nseq, max_seqlen, total_T, Hq, Hkv, d, causal, scale, stream);
}

fa_status_t fa_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* q_scale, const float* k_scale,
                       const float* v_scale, void* o, float* lse, int B, int Hq, int Hkv, int N, int d, int causal,
                       float scale, void* stream) {
  if (B < 0 || N < 0) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * N == 0) return FA_OK;
  if (static_cast<long long>(B) * N > INT32_MAX) return FA_ERR_UNSUPPORTED;
  fa_status_t st = check_common(q8, k8, v8, o, lse, Hq, Hkv, d, scale);
  if (st != FA_OK) return st;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if (!q_scale || !k_scale || !v_scale || !aligned(q_scale, 4) || !aligned(k_scale, 4) || !aligned(v_scale, 4))
    return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  if ((st = device_state(&ds)) != FA_OK) return st;
  fa::FwdArgs a{};
  a.o = o;
  a.lse = lse;
  a.cu_seqlens = nullptr;
  a.nseq = B;
  a.N = N;
  a.total_T = B * N;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.causal = causal;
  a.scale = scale;
  a.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  a.lse_head_stride = N;
  a.q_scale = q_scale;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.nblk_s = (N + 127) / 128;
  const long long bound = static_cast<long long>(B) * Hq * ((N + 255) / 256);
  if (bound > INT32_MAX) return FA_ERR_UNSUPPORTED;
  a.num_units = static_cast<int>(bound);
  // exponentials on MUFU only: the FMA pipe is shared with the V widening warps
  return launch_fwd<128, true>(ds, q8, k8, v8, a, B * N, bound, static_cast<cudaStream_t>(stream));
}

size_t fa_bwd_workspace_size(int tokens, int nseq, int Hq, int d) {
  (void)d;
  if (tokens <= 0 || Hq <= 0 || nseq < 0) return 0;
  return 2 * vec_bytes(tokens, nseq, Hq);
}

size_t fa_bwd_blocksparse_workspace_size(int B, int Hq, int Hkv, int N, int d) {
  if (B <= 0 || N <= 0 || Hq <= 0 || Hkv <= 0 || (d != 64 && d != 128)) return 0;
  if (static_cast<long long>(B) * N > INT32_MAX - 256) return 0;
  DeviceState* ds = nullptr;
  if (device_state(&ds) != FA_OK) return 0;
  return sparse_plan_layout(2 * vec_bytes(B * N, B, Hq), B, Hq, Hkv, N, d, ds->sms).total;
}

fa_status_t fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                   void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B, int Hq, int Hkv, int N,
                   int d, int causal, float scale, void* stream) {
  if (B < 0 || N < 0) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * N == 0) return FA_OK;
  if (static_cast<long long>(B) * N > INT32_MAX - 256) return FA_ERR_UNSUPPORTED;
  return bwd_dispatch(q, k, v, o, lse, dout, dq, dk, dv, workspace, ws_bytes, nullptr, B, N, B * N, Hq, Hkv, d,
                      causal, scale, stream);
}

fa_status_t fa_bwd_part(int parts, const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B,
                        int Hq, int Hkv, int N, int d, int causal, float scale, void* stream) {
  if (B < 0 || N < 0) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * N == 0) return FA_OK;
  if (static_cast<long long>(B) * N > INT32_MAX - 256) return FA_ERR_UNSUPPORTED;
  return bwd_dispatch(q, k, v, o, lse, dout, dq, dk, dv, workspace, ws_bytes, nullptr, B, N, B * N, Hq, Hkv, d,
                      causal, scale, stream, parts);
}

fa_status_t fa_bwd_fp8(const void* q8, const void* k8, const float* q_scale, const float* k_scale, const void* q,
                       const void* k, const void* v, const void* o, const float* lse, const void* dout, void* dq,
                       void* dk, void* dv, void* workspace, size_t ws_bytes, int B, int Hq, int Hkv, int N, int d,
                       int causal, float scale, void* stream) {
  if (B < 0 || N < 0) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * N == 0) return FA_OK;
  if (static_cast<long long>(B) * N > INT32_MAX - 256) return FA_ERR_UNSUPPORTED;
  if (!q8 || !k8 || !aligned(q8, 16) || !aligned(k8, 16)) return FA_ERR_INVALID_ARG;
  if (!q_scale || !k_scale || !aligned(q_scale, 4) || !aligned(k_scale, 4)) return FA_ERR_INVALID_ARG;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  return bwd_dispatch(q, k, v, o, lse, dout, dq, dk, dv, workspace, ws_bytes, nullptr, B, N, B * N, Hq, Hkv, d,
                      causal, scale, stream, FA_BWD_ALL, nullptr, q8, k8, q_scale, k_scale);
}

fa_status_t fa_bwd_blocksparse(const void* q, const void* k, const void* v, const unsigned char* block_mask,
                               const void* o, const float* lse, const void* dout, void* dq, void* dk, void* dv,
                               void* workspace, size_t ws_bytes, int B, int Hq, int Hkv, int N, int d, int causal,
                               float scale, void* stream) {
  if (B < 0 || N < 0) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * N == 0) return FA_OK;
  if (block_mask == nullptr) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * N > INT32_MAX - 256) return FA_ERR_UNSUPPORTED;
  return bwd_dispatch(q, k, v, o, lse, dout, dq, dk, dv, workspace, ws_bytes, nullptr, B, N, B * N, Hq, Hkv, d,
                      causal, scale, stream, FA_BWD_ALL, block_mask);
}

fa_status_t fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                          const void* dout, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                          const int* cu_seqlens, int nseq, int max_seqlen, int total_T, int Hq, int Hkv, int d,
                          int causal, float scale, void* stream) {
  if (nseq < 0 || total_T < 0 || max_seqlen < 0 || cu_seqlens == nullptr || !aligned(cu_seqlens, 4))
    return FA_ERR_INVALID_ARG;
  if (nseq == 0 || total_T == 0 || max_seqlen == 0) return FA_OK;
  if (max_seqlen > 131072 || total_T > INT32_MAX - 256) return FA_ERR_UNSUPPORTED;
  return bwd_dispatch(q, k, v, o, lse, dout, dq, dk, dv, workspace, ws_bytes, cu_seqlens, nseq, max_seqlen, total_T,
                      Hq, Hkv, d, causal, scale, stream);
}

fa_status_t fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                           const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d,
                           int causal, float scale, void* stream) {
  if (B < 0 || N < 0 || Hq <= 0) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * N == 0) return FA_OK;
  if (static_cast<long long>(B) * N > INT32_MAX - 256) return FA_ERR_UNSUPPORTED;
  // the whole working set must fit the built-in array
  const size_t need = fa_bwd_workspace_size(B * N, B, Hq, d);
  if (need > kNoAllocScratchBytes) return FA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const fa_status_t st = noalloc_scratch_address(&scratch);
  if (st != FA_OK) return st;
  // Nothing in the scratch has to start at zero: the first kernel of the
  // backward writes every entry the later two read.
  return fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, scratch, need, B, Hq, Hkv, N, d, causal, scale, stream);
}

size_t fa_fwd_kvcache_workspace_size(int B, int Nq, int Hq, int d, int num_splits) {
  if (B <= 0 || Nq <= 0 || Hq <= 0 || d <= 0 || num_splits <= 1) return 0;
  return dec_part_floats(B, Nq, Hq, d, num_splits) * sizeof(float);
}

int fa_fwd_kvcache_num_splits(int B, int Hkv, int Ncache, int d) {
  if (B <= 0 || Hkv <= 0 || Ncache <= 0 || (d != 64 && d != 128)) return 1;
  DeviceState* ds = nullptr;
  if (device_state(&ds) != FA_OK) return 1;
  // Launch-time model of the decode kernel, its constants measured on B200:
  // one CTA streams a 128-key tile in about t_tile when HBM is not the limit,
  // pays about t_unit per (sequence, kv head, split) unit, and the whole cache
  // cannot stream faster than the HBM rate; more than one split adds the
  // merge kernel. The persistent CTAs take units round-robin.
  const double t_tile = d == 128 ? 1.07e-6 : 0.93e-6;
  const double t_unit = 5e-6, t_merge = 12e-6, hbm_bytes_per_s = 6.4e12;
  const int tiles = (Ncache + fa::kDecKeys - 1) / fa::kDecKeys;
  const long long bh = static_cast<long long>(B) * Hkv;
  const double t_hbm = 4.0 * static_cast<double>(bh) * Ncache * d / hbm_bytes_per_s;
  double best = 0;
  int best_s = 1;
  for (int s = 1; s <= tiles && s <= 256; ++s) {
    const int chunk = dec_chunk_keys(Ncache, s);
    const int splits = (Ncache + chunk - 1) / chunk;
    if (splits != s) continue;  // same launch as a smaller count
    const int per = chunk / fa::kDecKeys;
    const long long rounds = (bh * splits + ds->sms - 1) / ds->sms;
    const double t_cta = static_cast<double>(rounds) * (per * t_tile + t_unit);
    const double cost = (t_cta > t_hbm ? t_cta : t_hbm) + (splits > 1 ? t_merge : 0.0);
    if (s == 1 || cost < best * 0.99) {  // more splits only for a clear gain
      best = cost;
      best_s = splits;
    }
  }
  return best_s;
}

fa_status_t fa_fwd_kvcache(const void* q, const void* k_cache, const void* v_cache, const int* cache_seqlens,
                           void* o, float* lse, void* workspace, size_t ws_bytes, int B, int Nq, int Hq, int Hkv,
                           int Ncache, int d, int causal, float scale, int num_splits, void* stream) {
  if (B < 0 || Nq < 0 || Ncache < 0 || num_splits < 1) return FA_ERR_INVALID_ARG;
  if (B == 0 || Nq == 0) return FA_OK;
  fa_status_t st = check_common(q, k_cache, v_cache, o, lse, Hq, Hkv, d, scale);
  if (st != FA_OK) return st;
  if (cache_seqlens == nullptr || !aligned(cache_seqlens, 4) || Ncache == 0) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (Nq * (Hq / Hkv) > fa::kDecRows) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * Ncache > INT32_MAX || B > 65535 || Hkv > 65535) return FA_ERR_UNSUPPORTED;
  const int chunk = dec_chunk_keys(Ncache, num_splits);
  const int splits = (Ncache + chunk - 1) / chunk;  // no empty trailing splits
  if (static_cast<long long>(B) * Hkv * splits > INT32_MAX) return FA_ERR_UNSUPPORTED;
  if (splits > 1) {
    if (workspace == nullptr || !aligned(workspace, 16) ||
        ws_bytes < dec_part_floats(B, Nq, Hq, d, splits) * sizeof(float))
      return FA_ERR_WORKSPACE;
  }
  DeviceState* ds = nullptr;
  if ((st = device_state(&ds)) != FA_OK) return st;
  fa::DecArgs a{};
  a.q = q;
  a.cache_seqlens = cache_seqlens;
  a.o = o;
  a.lse = lse;
  a.B = B;
  a.Nq = Nq;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Ncache = Ncache;
  a.splits = splits;
  a.chunk = chunk;
  a.num_units = B * Hkv * splits;
  a.causal = causal;
  a.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  if (splits > 1) {
    a.part_o = static_cast<float*>(workspace);
    a.part_lse = a.part_o + static_cast<size_t>(splits) * B * Nq * Hq * d;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d == 128 ? launch_decode<128>(ds, k_cache, v_cache, a, s) : launch_decode<64>(ds, k_cache, v_cache, a, s);
}

fa_status_t fa_attn_merge(const void* o_parts, const float* lse_parts, int nparts, void* o, float* lse, int B, int N,
                          int H, int d, void* stream) {
  if (B < 0 || N < 0 || H <= 0 || nparts < 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return FA_OK;
  if (!o_parts || !lse_parts || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned(o_parts, 16) || !aligned(o, 16) || !aligned(lse_parts, 4) || !aligned(lse, 4))
    return FA_ERR_INVALID_ARG;
  fa::MergeArgs a{};
  a.o_parts = o_parts;
  a.lse_parts = lse_parts;
  a.o = o;
  a.lse = lse;
  a.rows = static_cast<long long>(B) * N * H;
  a.N = N;
  a.H = H;
  a.nparts = nparts;
  const long long rows_per_block = 8LL * (32 / (d / 8));  // 8 warps, 32/(d/8) rows each
  const long long blocks = (a.rows + rows_per_block - 1) / rows_per_block;
  if (blocks > INT32_MAX) return FA_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 128)
    fa::fa_merge_kernel<128><<<static_cast<int>(blocks), 256, 0, s>>>(a);
  else
    fa::fa_merge_kernel<64><<<static_cast<int>(blocks), 256, 0, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status_t fa_fp8_quantize(const void* x, void* codes, float* scales, int B, int N, int H, int d, int rotate,
                            void* stream) {
  if (B < 0 || N < 0 || H <= 0 || (rotate != 0 && rotate != 1)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return FA_OK;
  if (!x || !codes || !scales || !aligned(x, 8) || !aligned(codes, 4) || !aligned(scales, 4))
    return FA_ERR_INVALID_ARG;
  const int nblk = (N + 127) / 128;
  if (B > 65535 || H > 65535) return FA_ERR_UNSUPPORTED;
  fa::QuantArgs a{};
  a.x = x;
  a.codes = static_cast<uint8_t*>(codes);
  a.scales = scales;
  a.B = B;
  a.N = N;
  a.H = H;
  a.nblk = nblk;
  a.rotate = rotate;
  a.rscale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
  dim3 grid(nblk, H, B);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 128)
    fa::fa_quant_kernel<128><<<grid, 256, 0, s>>>(a);
  else
    fa::fa_quant_kernel<64><<<grid, 256, 0, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status_t fa_fp8_dequantize(const void* codes, const float* scales, void* x, int B, int N, int H, int d,
                              int unrotate, void* stream) {
  if (B < 0 || N < 0 || H <= 0 || (unrotate != 0 && unrotate != 1)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return FA_OK;
  if (!x || !codes || !scales || !aligned(x, 8) || !aligned(codes, 4) || !aligned(scales, 4))
    return FA_ERR_INVALID_ARG;
  const int nblk = (N + 127) / 128;
  if (B > 65535 || H > 65535) return FA_ERR_UNSUPPORTED;
  fa::DequantArgs a{};
  a.codes = static_cast<const uint8_t*>(codes);
  a.scales = scales;
  a.x = x;
  a.B = B;
  a.N = N;
  a.H = H;
  a.nblk = nblk;
  a.unrotate = unrotate;
  a.rscale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
  dim3 grid(nblk, H, B);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 128)
    fa::fa_dequant_kernel<128><<<grid, 256, 0, s>>>(a);
  else
    fa::fa_dequant_kernel<64><<<grid, 256, 0, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status_t fa_grad_accumulate(float* acc, const void* part, void* out, long long count, int first, void* stream) {
  if (count < 0 || count % 8 != 0 || (first != 0 && first != 1)) return FA_ERR_INVALID_ARG;
  if (count == 0) return FA_OK;
  if (!acc || !aligned(acc, 16) || (part && !aligned(part, 16)) || (out && !aligned(out, 16)))
    return FA_ERR_INVALID_ARG;
  fa::AccArgs a{};
  a.acc = acc;
  a.part = part;
  a.out = out;
  a.n8 = count / 8;
  a.first = first;
  const long long blocks = (a.n8 + 255) / 256;
  if (blocks > INT32_MAX) return FA_ERR_UNSUPPORTED;
  fa::fa_grad_accumulate_kernel<<<static_cast<int>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status_t fa_get_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  int w = 0;
  if (cudaMemcpyFromSymbol(&w, g_status_word, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (w == 0) return FA_OK;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  g_last_word.store(w);
  return static_cast<fa_status_t>(w & 0xff);
}

int fa_last_device_error_word(void) { return g_last_word.load(); }

const char* fa_status_string(fa_status_t s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
  }
  return "FA_ERR_UNKNOWN";
}

void fa_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns.store(ns == 0 ? 1 : ns); }

void fa_debug_set_inject(int mode) { g_inject.store(mode); }

}  // extern "C"
