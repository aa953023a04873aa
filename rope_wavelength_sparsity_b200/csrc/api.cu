// C ABI of the windowed-attention library (declarations and contracts in
// include/wpattn.h).  Host side: argument checks, the planner, TMA tensor
// maps and kernel launches.  Every step of the computation runs in the
// kernels of decode_kernels.cuh and prefill_kernel.cuh.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "wpattn.h"
#include "planner.h"
#include "device_util.cuh"
#include "decode_kernels.cuh"
#include "prefill_kernel.cuh"
#include "rope_kernels.cuh"

namespace wpattn {
namespace {

constexpr int kMaxDevices = 64;

// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library links no libcuda and loads on hosts without a GPU driver.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

struct DeviceInfo {
  bool init = false;
  bool supported = false;
  int num_sms = 0;
  int decode_slots = 0;  // decode CTAs resident on the whole GPU at once
  // shared-memory attribute set, per prefill instantiation: (D 64, 128) x (g 1, 8) x
  // (plain, block mask, positions); atomic because host threads may launch concurrently
  std::atomic<bool> prefill_attr[16] = {};
  void* static_scratch = nullptr;  // device address of g_decode_static_scratch
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WPATTN_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return WPATTN_EUNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.init) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return WPATTN_ECUDA;
    d.supported = (major == 10 && minor == 0);
    d.num_sms = sms;
    if (d.supported) {
      // resident decode CTAs per SM, limited by the shared-memory ring and by
      // the registers of the largest instantiation
      int smem_sm = 0, smem_res = 0, regs_sm = 0;
      cudaFuncAttributes fa;
      if (cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&smem_res, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev) != cudaSuccess ||
          cudaFuncGetAttributes(&fa, decode_split_kernel<128, 8, false>) != cudaSuccess)
        return WPATTN_ECUDA;
      const int cta_smem = std::max(DecodeSmem<64>::ALLOC, DecodeSmem<128>::ALLOC) + smem_res;
      const int warps = kDecodeComputeWarps + 1;
      const int cta_regs = warps * ((fa.numRegs * 32 + 255) / 256 * 256);
      int per_sm = std::min(smem_sm / cta_smem, cta_regs > 0 ? regs_sm / cta_regs : 1);
      if (per_sm < 1) per_sm = 1;
      d.decode_slots = sms * per_sm;
    }
    d.init = true;
  }
  *out = &d;
  return d.supported ? WPATTN_OK : WPATTN_EUNSUPPORTED;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// bf16 tensor map with explicit byte strides of dims 1..3 (dim 0 contiguous), no swizzle
int encode_bf16_4d_strided(CUtensorMap* map, const void* base, const cuuint64_t (&dims)[4],
                           const cuuint64_t (&strides)[3], uint32_t box0, uint32_t box1) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return WPATTN_ECUDA;
  const cuuint32_t box[4] = {box0, box1, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? WPATTN_OK : WPATTN_ECUDA;
}

// bf16 tensor map of a [d3, d1, d2, d0] tensor (d0 contiguous), L2 misses
// widened to 256 bytes (whole rows of a head)
int encode_bf16_4d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                   uint64_t d3, uint32_t box0, uint32_t box1, bool swizzle128) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return WPATTN_ECUDA;
  const cuuint64_t dims[4] = {d0, d1, d2, d3};
  const cuuint64_t strides[3] = {d0 * d2 * 2, d0 * 2, d0 * d1 * d2 * 2};  // row, head, batch
  const cuuint32_t box[4] = {box0, box1, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? WPATTN_OK : WPATTN_ECUDA;
}

// theta_p = base^(-2p/D), the RoPE angle per position of pair p
void rope_thetas(double base, int D, double* theta) {
  for (int p = 0; p < 64; ++p)
    theta[p] = p < D / 2 ? std::pow(base, -static_cast<double>(2 * p) / static_cast<double>(D)) : 0.0;
}

// Rotation of one tensor, or of two in one launch (x1 null for one).  Every
// tensor has B sequences and the same head dim D.
int launch_rope(const void* x0, void* out0, int64_t N0, int H0, int64_t pos0_0, const int32_t* pos,
                const void* x1, void* out1, int64_t N1, int H1, int64_t pos0_1, int64_t B, int D,
                double base, int num_sms, cudaStream_t st) {
  RopeParams rp;
  std::memset(&rp, 0, sizeof rp);
  rp.seg[0] = RopeSegment{static_cast<const uint16_t*>(x0), static_cast<uint16_t*>(out0), pos, pos0_0,
                          N0, H0};
  rp.nseg = 1;
  if (x1 && N1 > 0) {
    rp.seg[1] = RopeSegment{static_cast<const uint16_t*>(x1), static_cast<uint16_t*>(out1), nullptr,
                            pos0_1, N1, H1};
    rp.nseg = 2;
  }
  rope_thetas(base, D, rp.theta);
  // (token, 8-pair chunk) items
  rp.items0 = static_cast<uint64_t>(B) * N0 * (D / 16);
  rp.items = rp.items0 + (rp.nseg == 2 ? static_cast<uint64_t>(B) * N1 * (D / 16) : 0);
  if (rp.items == 0) return WPATTN_OK;
  const uint64_t want = (rp.items + 255) / 256;
  const unsigned grid = static_cast<unsigned>(std::min<uint64_t>(want, static_cast<uint64_t>(num_sms) * 8));
  if (D == 64) rope_kernel<64><<<grid, 256, 0, st>>>(rp);
  else rope_kernel<128><<<grid, 256, 0, st>>>(rp);
  return cudaGetLastError() == cudaSuccess ? WPATTN_OK : WPATTN_ECUDA;
}

template <int D, bool G8, bool MASK, bool POS, bool SPLIT = false>
int launch_prefill(const void* q, const void* k, const void* v, PrefillParams prm,
                   DeviceInfo* dev, cudaStream_t st) {
  using Shape = PrefillShape<D>;
  CUtensorMap tq, tk, tv;
  int rc;
  prm.num_ctas_q = (prm.Nq + Shape::QT * kBM - 1) / (Shape::QT * kBM);
  // tensors are [B, N, H, D]: dims (fastest first) D, N, H, B
  if ((rc = encode_bf16_4d(&tq, q, D, prm.Nq, prm.Hq, prm.B, 8, kBM, false)) != WPATTN_OK) return rc;
  // with no key the kernel issues no K/V load; the maps only need to be valid
  const uint64_t nk = prm.Nk > 0 ? prm.Nk : prm.Nq;
  const uint64_t hk = prm.Nk > 0 ? prm.Hkv : prm.Hq;
  if ((rc = encode_bf16_4d(&tk, k, D, nk, hk, prm.B, 8, Shape::BN, false)) != WPATTN_OK) return rc;
  if ((rc = encode_bf16_4d(&tv, v, D, nk, hk, prm.B, 64, Shape::BN, true)) != WPATTN_OK) return rc;
  constexpr int smem = PrefillSmem<D>::ALLOC;
  const int slot = SPLIT ? 12 + (D == 64 ? 0 : 2) + (G8 ? 1 : 0)
                         : (D == 64 ? 0 : 6) + (G8 ? 3 : 0) + (MASK ? 1 : 0) + (POS ? 2 : 0);
  // a mask bit covers one 128-row query tile x one 128-key tile
  if (MASK && (Shape::BN != 128 || kBM != 128)) return WPATTN_EUNSUPPORTED;
  if (!dev->prefill_attr[slot].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(prefill_kernel<D, G8, MASK, POS, SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
      return WPATTN_ECUDA;
    dev->prefill_attr[slot].store(true, std::memory_order_release);
  }
  if constexpr (SPLIT) {
    // the split items' parts, then their merge
    const dim3 grid(static_cast<unsigned>(prm.split_items) * prm.kv_splits);
    prefill_kernel<D, G8, MASK, POS, true><<<grid, Shape::THREADS, smem, st>>>(tq, tk, tv, prm);
    if (cudaGetLastError() != cudaSuccess) return WPATTN_ECUDA;
    prefill_combine_kernel<D><<<static_cast<unsigned>(prm.split_items) * Shape::QT * kBM, D, 0, st>>>(prm);
  } else {
    const dim3 grid = prm.heads_fast ? dim3(prm.Hq, prm.B, prm.num_ctas_q) : dim3(prm.num_ctas_q, prm.Hq, prm.B);
    prefill_kernel<D, G8, MASK, POS, false><<<grid, Shape::THREADS, smem, st>>>(tq, tk, tv, prm);
  }
  return cudaGetLastError() == cudaSuccess ? WPATTN_OK : WPATTN_ECUDA;
}

template <int D, bool MASK, bool POS, bool SPLIT = false>
int launch_prefill_g(const void* q, const void* k, const void* v, const PrefillParams& prm,
                     DeviceInfo* dev, cudaStream_t st) {
  return prm.g8 ? launch_prefill<D, true, MASK, POS, SPLIT>(q, k, v, prm, dev, st)
                : launch_prefill<D, false, MASK, POS, SPLIT>(q, k, v, prm, dev, st);
}

template <int D>
int launch_prefill_mode(const void* q, const void* k, const void* v, const PrefillParams& prm,
                        DeviceInfo* dev, cudaStream_t st) {
  if (prm.block_mask && prm.q_pos) return WPATTN_EUNSUPPORTED;
  if (prm.kv_splits > 1) {
    // the unsplit kernel takes the items below item_end (full waves), the split
    // kernel the rest
    if (prm.block_mask || prm.q_pos) return WPATTN_EUNSUPPORTED;
    int rc = WPATTN_OK;
    if (prm.item_end > 0) rc = launch_prefill_g<D, false, false, false>(q, k, v, prm, dev, st);
    if (rc != WPATTN_OK) return rc;
    return launch_prefill_g<D, false, false, true>(q, k, v, prm, dev, st);
  }
  if (prm.block_mask) return launch_prefill_g<D, true, false>(q, k, v, prm, dev, st);
  if (prm.q_pos) return launch_prefill_g<D, false, true>(q, k, v, prm, dev, st);
  return launch_prefill_g<D, false, false>(q, k, v, prm, dev, st);
}

template <int D, int GC, bool PM>
int launch_decode_split(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& prm,
                        cudaStream_t st) {
  constexpr int smem = DecodeSmem<D>::ALLOC;
  static std::atomic<bool> attr_set[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WPATTN_ECUDA;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(decode_split_kernel<D, GC, PM>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return WPATTN_ECUDA;
    attr_set[dev].store(true, std::memory_order_release);
  }
  dim3 grid(prm.S, prm.Hkv * prm.hchunks, prm.B);
  decode_split_kernel<D, GC, PM><<<grid, (kDecodeComputeWarps + 1) * 32, smem, st>>>(tk, tv, prm);
  return cudaGetLastError() == cudaSuccess ? WPATTN_OK : WPATTN_ECUDA;
}

template <int D, bool PM>
int launch_decode_gc(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& prm, int gc,
                     cudaStream_t st) {
  switch (gc) {
    case 1: return launch_decode_split<D, 1, PM>(tk, tv, prm, st);
    case 2: return launch_decode_split<D, 2, PM>(tk, tv, prm, st);
    case 3: return launch_decode_split<D, 3, PM>(tk, tv, prm, st);
    case 4: return launch_decode_split<D, 4, PM>(tk, tv, prm, st);
    case 5: return launch_decode_split<D, 5, PM>(tk, tv, prm, st);
    case 6: return launch_decode_split<D, 6, PM>(tk, tv, prm, st);
    case 7: return launch_decode_split<D, 7, PM>(tk, tv, prm, st);
    case 8: return launch_decode_split<D, 8, PM>(tk, tv, prm, st);
    default: return WPATTN_EUNSUPPORTED;
  }
}

template <int D>
int launch_decode(const DecodeParams& prm, int gc, bool pm, cudaStream_t st) {
  int rc;
  CUtensorMap tk, tv;
  constexpr uint32_t KB = DecodeSmem<D>::KB;
  if (pm) {
    // pair-major K slabs [B, Hkv, D/16, Lmax, 16]: dims (fastest first) 16, Lmax,
    // Hkv * D/16 (slab planes), B; 16-dim x 32-key boxes
    const uint64_t planes = static_cast<uint64_t>(prm.Hkv) * (D / 16);
    const cuuint64_t dims[4] = {16, static_cast<cuuint64_t>(prm.Lmax), planes, static_cast<cuuint64_t>(prm.B)};
    const cuuint64_t strides[3] = {32, static_cast<cuuint64_t>(prm.Lmax) * 32,
                                   planes * static_cast<cuuint64_t>(prm.Lmax) * 32};
    if ((rc = encode_bf16_4d_strided(&tk, prm.k, dims, strides, 16, KB)) != WPATTN_OK) return rc;
  } else if (prm.block_table) {
    // page pools [num_pages, page_size, Hkv, D]: dims D, page_size, Hkv, num_pages;
    // boxes of 64 dims x min(page_size, 32) rows (a copy never crosses a page)
    const uint32_t R = prm.page_size < static_cast<int>(KB) ? prm.page_size : KB;
    if ((rc = encode_bf16_4d(&tk, prm.k, D, prm.page_size, prm.Hkv, prm.num_pages, 64, R, true)) != WPATTN_OK)
      return rc;
    if ((rc = encode_bf16_4d(&tv, prm.v, D, prm.page_size, prm.Hkv, prm.num_pages, 64, R, true)) != WPATTN_OK)
      return rc;
  } else {
    // caches are [B, Lmax, Hkv, D]: dims (fastest first) D, Lmax, Hkv, B; 64-dim x 32-key boxes
    if ((rc = encode_bf16_4d(&tk, prm.k, D, prm.Lmax, prm.Hkv, prm.B, 64, KB, true)) != WPATTN_OK)
      return rc;
  }
  if (!prm.block_table &&
      (rc = encode_bf16_4d(&tv, prm.v, D, prm.Lmax, prm.Hkv, prm.B, 64, KB, true)) != WPATTN_OK)
    return rc;
  rc = pm ? launch_decode_gc<D, true>(tk, tv, prm, gc, st) : launch_decode_gc<D, false>(tk, tv, prm, gc, st);
  if (rc != WPATTN_OK) return rc;
  const size_t smem = static_cast<size_t>(prm.S) * 2 * sizeof(float);
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(decode_combine_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return WPATTN_ECUDA;
  }
  decode_combine_kernel<D><<<prm.B * prm.Hq, D, smem, st>>>(prm);
  return cudaGetLastError() == cudaSuccess ? WPATTN_OK : WPATTN_ECUDA;
}

}  // namespace
}  // namespace wpattn

// Scratch for wpattn_decode_noalloc: a fixed-size array in the library's own
// device image, so that entry point never allocates.  Every GPU that loads
// the library holds these bytes until the process exits.
constexpr size_t kDecodeStaticScratchBytes = size_t(4) << 20;  // 4 MiB
static __device__ __align__(256) unsigned char g_decode_static_scratch[kDecodeStaticScratchBytes];

namespace wpattn {
// One thread waits on an mbarrier that nothing arrives at: the bounded wait
// runs out, records WPATTN_ETIMEOUT and the kernel returns (the failure path
// of every wait in the library's kernels, exercised without a fault).
__global__ void selftest_wait_kernel() {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(b, 0);
  __syncthreads();
}
}  // namespace wpattn

using namespace wpattn;

extern "C" {

const char* wpattn_version(void) { return "0.1.0"; }

const char* wpattn_strerror(int code) {
  switch (code) {
    case WPATTN_OK: return "ok";
    case WPATTN_EINVAL: return "invalid argument";
    case WPATTN_EUNSUPPORTED: return "unsupported configuration or device";
    case WPATTN_ECUDA: return "CUDA runtime or launch error";
    case WPATTN_ETIMEOUT: return "a kernel gave up a bounded wait";
    case WPATTN_EWORKSPACE: return "workspace missing or too small";
    case WPATTN_EINDEX: return "a device-side index (page or position) was out of range";
    default: return "unknown status code";
  }
}

int wpattn_thresholds(const wpattn_window* w, int64_t* T_eff) {
  if (!w || !T_eff) return WPATTN_EINVAL;
  WindowPlan plan;
  const int rc = make_window_plan(w, &plan);
  if (rc == WPATTN_EUNSUPPORTED) {
    // wide head dims: host-only evaluation
    for (int p = 0; p < w->head_dim / 2; ++p) T_eff[p] = effective_threshold(w, p);
    return WPATTN_OK;
  }
  if (rc != WPATTN_OK) return rc;
  for (int p = 0; p < plan.P; ++p) T_eff[p] = plan.T[p];
  return WPATTN_OK;
}

int wpattn_pruned_fraction(const wpattn_window* w, int64_t Nq, int64_t Nk, int64_t q_pos0,
                           int64_t k_pos0, uint64_t* pruned_terms, uint64_t* total_terms,
                           double* fraction) {
  if (!w || Nq < 0 || Nk < 0) return WPATTN_EINVAL;
  WindowPlan plan;
  const int rc = make_window_plan(w, &plan);
  if (rc != WPATTN_OK && rc != WPATTN_EUNSUPPORTED) return rc;
  const int P = w->head_dim / 2;
  // causal (query, key) pairs = kept terms of a pair whose threshold never binds
  const unsigned __int128 causal = kept_terms_one_pair(kNoLimit, Nq, Nk, q_pos0, k_pos0);
  unsigned __int128 kept = 0;
  for (int p = 0; p < P; ++p) kept += kept_terms_one_pair(effective_threshold(w, p), Nq, Nk, q_pos0, k_pos0);
  const unsigned __int128 total = causal * static_cast<unsigned __int128>(P);
  const unsigned __int128 pruned = total - kept;
  if ((total >> 64) != 0) return WPATTN_EUNSUPPORTED;  // beyond 64-bit counts
  if (pruned_terms) *pruned_terms = static_cast<uint64_t>(pruned);
  if (total_terms) *total_terms = static_cast<uint64_t>(total);
  if (fraction) *fraction = total ? static_cast<double>(pruned) / static_cast<double>(total) : 0.0;
  return WPATTN_OK;
}

}  // extern "C"

namespace {
constexpr int kPrefillBN = 128;  // keys per key tile of the prefill kernel (both head dims)
static_assert(PrefillShape<64>::BN == kPrefillBN && PrefillShape<128>::BN == kPrefillBN,
              "the split plan counts key tiles of 128 keys");

constexpr int kItemRows = 256;   // query rows of one work item (two 128-row tiles)

// Which work items (CTAs of the unsplit grid) run with their key range split,
// and into how many parts: main_items run unsplit, the split_items after
// them as parts of per key tiles each.
struct SplitPlan {
  int64_t items = 0, main_items = 0;
  int split_items = 0, parts = 1, per = 0;
  size_t bytes(int D) const {   // fp32 O parts, then the parts' log2-sum-exps
    return split_items > 0 ? static_cast<size_t>(parts) * split_items * kItemRows * (D + 1) * sizeof(float)
                           : 0;
  }
};

// kv_splits >= 2: every item in kv_splits parts.  kv_splits == 0: when every
// item does about the same work (the last query sees at most 10% more keys
// than the first, as for a chunk far into a long context), the items of the
// grid's last partial wave (one CTA per SM) are split into min(8, num_sms /
// their count) parts of at least 64 key tiles, so that they finish in a
// fraction of a wave.  Otherwise (and for kv_splits == 1) nothing is split.
SplitPlan make_split_plan(int64_t B, int64_t Nq, int64_t Nk, int64_t Hq, int64_t qk_off,
                          int kv_splits, int num_sms) {
  SplitPlan sp;
  sp.items = (Nq + kItemRows - 1) / kItemRows * Hq * B;
  sp.main_items = sp.items;
  if (B <= 0 || Nq <= 0 || Nk <= 0 || Hq <= 0 || kv_splits == 1) return sp;
  const int64_t nkt = (Nk + kPrefillBN - 1) / kPrefillBN;
  int S = kv_splits;
  int64_t first_split = 0;
  if (kv_splits == 0) {
    const int64_t first = std::min<int64_t>(std::max<int64_t>(qk_off + 1, 0), Nk);
    const int64_t last = std::min<int64_t>(std::max<int64_t>(qk_off + Nq, 0), Nk);
    if (num_sms <= 0 || last <= 0 || first * 10 < last * 9) return sp;
    const int64_t r = sp.items % num_sms;
    if (r == 0) return sp;
    S = static_cast<int>(std::min<int64_t>(8, num_sms / r));
    S = static_cast<int>(std::min<int64_t>(S, ((last + kPrefillBN - 1) / kPrefillBN) / 64));
    if (S < 2) return sp;
    first_split = sp.items - r;
  }
  const int64_t per = (nkt + S - 1) / S;
  S = static_cast<int>((nkt + per - 1) / per);   // no part past the last key tile
  if (S < 2) return sp;
  sp.main_items = first_split;
  sp.split_items = static_cast<int>(sp.items - first_split);
  sp.parts = S;
  sp.per = static_cast<int>(per);
  return sp;
}

// wpattn_prefill and wpattn_prefill_masked: block_mask null = no mask
int prefill_impl(const wpattn_window* w, const void* q, const void* k, const void* v, void* out,
                 float* lse, int32_t B, int32_t Nq, int32_t Nk, int32_t Hq, int32_t Hkv,
                 int64_t q_pos0, int64_t k_pos0, float softmax_scale, const uint32_t* block_mask,
                 int32_t mask_words, void* cuda_stream, const int32_t* q_pos = nullptr,
                 int64_t q_pos_stride = 0, const int32_t* k_pos = nullptr,
                 int64_t k_pos_stride = 0, int32_t kv_splits = 1, void* workspace = nullptr,
                 size_t workspace_bytes = 0) {
  WindowPlan plan;
  int rc = make_window_plan(w, &plan);
  if (rc != WPATTN_OK) return rc;
  if (B < 0 || Nq < 0 || Nk < 0 || Hq <= 0 || Hkv <= 0 || (Hq % Hkv) != 0) return WPATTN_EINVAL;
  if (!(softmax_scale == softmax_scale)) return WPATTN_EINVAL;  // NaN
  if (plan.D != 64 && plan.D != 128) return WPATTN_EUNSUPPORTED;
  if (B == 0 || Nq == 0) return WPATTN_OK;
  if (!q || !out || (Nk > 0 && (!k || !v))) return WPATTN_EINVAL;
  if (!aligned16(q) || !aligned16(out) || (Nk > 0 && (!aligned16(k) || !aligned16(v))))
    return WPATTN_EINVAL;
  // positions must keep every distance well inside int64
  if (q_pos0 < 0 || k_pos0 < 0 || q_pos0 > (int64_t(1) << 60) || k_pos0 > (int64_t(1) << 60))
    return WPATTN_EINVAL;
  if (static_cast<int64_t>(B) * Hq > 65535LL * 65535LL || Hq > 65535 || B > 65535)
    return WPATTN_EUNSUPPORTED;
  DeviceInfo* dev = nullptr;
  if ((rc = device_info(&dev)) != WPATTN_OK) return rc;

  PrefillParams prm;
  std::memset(&prm, 0, sizeof prm);
  prm.out = static_cast<uint16_t*>(out);
  prm.lse = lse;
  prm.B = B; prm.Nq = Nq; prm.Nk = Nk; prm.Hq = Hq; prm.Hkv = Hkv; prm.G = Hq / Hkv;
  // the kernel works in positions relative to k_pos0, in 32-bit integers
  const int64_t qk_off = q_pos0 - k_pos0;
  if (qk_off < -(int64_t(1) << 30) || qk_off > (int64_t(1) << 30) || Nq > (1 << 30) ||
      Nk > (1 << 30))
    return WPATTN_EUNSUPPORTED;
  prm.qk_off = static_cast<int>(qk_off);
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(plan.D));
  prm.scale_log2 = scale * 1.44269504088896340736f;
  prm.g8 = plan.g == 8 ? 1 : 0;
  if (q_pos) {
    // k_pos rows travel to shared memory 128 keys at a time by bulk copy
    const int64_t padded = (static_cast<int64_t>(Nk) + 127) / 128 * 128;
    if (!k_pos || q_pos_stride < Nq || k_pos_stride < padded || (k_pos_stride & 3) != 0 ||
        (reinterpret_cast<uintptr_t>(q_pos) & 3u) != 0 || (reinterpret_cast<uintptr_t>(k_pos) & 15u) != 0)
      return WPATTN_EINVAL;
    prm.q_pos = q_pos;
    prm.k_pos = k_pos;
    prm.q_pos_stride = q_pos_stride;
    prm.k_pos_stride = k_pos_stride;
  }
  if (block_mask) {
    const int64_t nkt = (static_cast<int64_t>(Nk) + 127) / 128;
    if (mask_words < (nkt + 31) / 32 || (reinterpret_cast<uintptr_t>(block_mask) & 3u) != 0)
      return WPATTN_EINVAL;
    prm.block_mask = block_mask;
    prm.mask_words = mask_words;
  }
  for (int p = 0; p < 64; ++p) prm.T[p] = plan.T[p] > INT32_MAX ? INT32_MAX : static_cast<int>(plan.T[p]);
  prm.item_end = INT64_MAX;
  if (kv_splits != 1) {
    const SplitPlan sp = make_split_plan(B, Nq, Nk, Hq, qk_off, kv_splits, dev->num_sms);
    if (sp.split_items > 0) {
      if (sp.items > 0x7FFFFFFFLL ||
          static_cast<int64_t>(sp.split_items) * std::max(sp.parts, kItemRows) > 0x7FFFFFFFLL)
        return WPATTN_EUNSUPPORTED;
      if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return WPATTN_EINVAL;
      if (workspace_bytes < sp.bytes(plan.D)) return WPATTN_EWORKSPACE;
      prm.item_end = sp.main_items;
      prm.split_item0 = static_cast<int>(sp.main_items);
      prm.split_items = sp.split_items;
      prm.kv_splits = sp.parts;
      prm.split_tiles = sp.per;
      prm.part_o = static_cast<float*>(workspace);
      prm.part_l = prm.part_o + static_cast<size_t>(sp.parts) * sp.split_items * kItemRows * plan.D;
    }
  }
  // Heaviest query blocks of every head first when the whole K and V stay in L2
  // (concurrent CTAs of many heads then share no L2 working set they would
  // thrash); otherwise one head's blocks after another, so that concurrent CTAs
  // walk the same K and V.
  {
    const int64_t nq_ctas = (static_cast<int64_t>(Nq) + 255) / 256;
    const int64_t kv_bytes = static_cast<int64_t>(B) * Nk * Hkv * plan.D * 4;
    prm.heads_fast = (prm.g8 && prm.item_end == INT64_MAX && nq_ctas <= 65535 &&
                      kv_bytes <= (int64_t(48) << 20)) ? 1 : 0;
  }
  const void* kk = Nk > 0 ? k : q;
  const void* vv = Nk > 0 ? v : q;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  if (plan.D == 64)
    return launch_prefill_mode<64>(q, kk, vv, prm, dev, st);
  return launch_prefill_mode<128>(q, kk, vv, prm, dev, st);
}

}  // namespace

extern "C" {

int wpattn_prefill(const wpattn_window* w, const void* q, const void* k, const void* v, void* out,
                   float* lse, int32_t B, int32_t Nq, int32_t Nk, int32_t Hq, int32_t Hkv,
                   int64_t q_pos0, int64_t k_pos0, float softmax_scale, void* cuda_stream) {
  return prefill_impl(w, q, k, v, out, lse, B, Nq, Nk, Hq, Hkv, q_pos0, k_pos0, softmax_scale,
                      nullptr, 0, cuda_stream);
}

int wpattn_prefill_split_plan(int32_t B, int32_t Nq, int32_t Nk, int32_t Hq, int64_t q_pos0,
                              int64_t k_pos0, int32_t kv_splits, int32_t num_sms, int64_t* main_items,
                              int32_t* split_items, int32_t* parts) {
  if (B < 0 || Nq < 0 || Nk < 0 || Hq <= 0 || kv_splits < 0 || kv_splits > 64) return WPATTN_EINVAL;
  if (num_sms <= 0) {
    DeviceInfo* dev = nullptr;
    const int rc = device_info(&dev);
    if (rc != WPATTN_OK) return rc;
    num_sms = dev->num_sms;
  }
  const SplitPlan sp = make_split_plan(B, Nq, Nk, Hq, q_pos0 - k_pos0, kv_splits, num_sms);
  if (main_items) *main_items = sp.main_items;
  if (split_items) *split_items = sp.split_items;
  if (parts) *parts = sp.split_items > 0 ? sp.parts : 1;
  return WPATTN_OK;
}

size_t wpattn_prefill_split_workspace_size(int32_t B, int32_t Nq, int32_t Nk, int32_t Hq,
                                           int32_t head_dim, int64_t q_pos0, int64_t k_pos0,
                                           int32_t kv_splits, int32_t num_sms) {
  if (B <= 0 || Nq <= 0 || Nk <= 0 || Hq <= 0 || (head_dim != 64 && head_dim != 128) ||
      kv_splits < 0 || kv_splits > 64)
    return 0;
  if (num_sms <= 0) {
    DeviceInfo* dev = nullptr;
    if (device_info(&dev) != WPATTN_OK) return 0;
    num_sms = dev->num_sms;
  }
  return make_split_plan(B, Nq, Nk, Hq, q_pos0 - k_pos0, kv_splits, num_sms).bytes(head_dim);
}

int wpattn_prefill_split(const wpattn_window* w, const void* q, const void* k, const void* v,
                         void* out, float* lse, int32_t B, int32_t Nq, int32_t Nk, int32_t Hq,
                         int32_t Hkv, int64_t q_pos0, int64_t k_pos0, float softmax_scale,
                         int32_t kv_splits, void* workspace, size_t workspace_bytes, void* cuda_stream) {
  if (kv_splits < 0 || kv_splits > 64) return WPATTN_EINVAL;
  return prefill_impl(w, q, k, v, out, lse, B, Nq, Nk, Hq, Hkv, q_pos0, k_pos0, softmax_scale,
                      nullptr, 0, cuda_stream, nullptr, 0, nullptr, 0, kv_splits, workspace,
                      workspace_bytes);
}

int wpattn_prefill_masked(const wpattn_window* w, const void* q, const void* k, const void* v,
                          void* out, float* lse, int32_t B, int32_t Nq, int32_t Nk, int32_t Hq,
                          int32_t Hkv, int64_t q_pos0, int64_t k_pos0, float softmax_scale,
                          const uint32_t* block_mask, int32_t mask_words, void* cuda_stream) {
  if (!block_mask) return WPATTN_EINVAL;
  return prefill_impl(w, q, k, v, out, lse, B, Nq, Nk, Hq, Hkv, q_pos0, k_pos0, softmax_scale,
                      block_mask, mask_words, cuda_stream);
}

int wpattn_prefill_positions(const wpattn_window* w, const void* q, const void* k, const void* v,
                             void* out, float* lse, int32_t B, int32_t Nq, int32_t Nk, int32_t Hq,
                             int32_t Hkv, const int32_t* q_pos, int64_t q_pos_stride,
                             const int32_t* k_pos, int64_t k_pos_stride, float softmax_scale,
                             void* cuda_stream) {
  if (!q_pos || !k_pos) return WPATTN_EINVAL;
  return prefill_impl(w, q, k, v, out, lse, B, Nq, Nk, Hq, Hkv, 0, 0, softmax_scale, nullptr, 0,
                      cuda_stream, q_pos, q_pos_stride, k_pos, k_pos_stride);
}

int wpattn_pack_block_mask(const uint8_t* mask, uint32_t* words, int64_t rows, int32_t nkb,
                           int32_t mask_words, void* cuda_stream) {
  if (rows < 0 || nkb < 0 || mask_words < (nkb + 31) / 32) return WPATTN_EINVAL;
  if (rows == 0 || mask_words == 0) return WPATTN_OK;
  if (!mask || !words || (reinterpret_cast<uintptr_t>(words) & 3u) != 0) return WPATTN_EINVAL;
  DeviceInfo* dev = nullptr;
  int rc;
  if ((rc = device_info(&dev)) != WPATTN_OK) return rc;
  const uint64_t n = static_cast<uint64_t>(rows) * static_cast<uint64_t>(mask_words);
  const uint64_t blocks = (n + 255) / 256;
  if (blocks > 0x7FFFFFFFull) return WPATTN_EUNSUPPORTED;
  pack_block_mask_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(cuda_stream)>>>(
      mask, words, rows, nkb, mask_words);
  return cudaGetLastError() == cudaSuccess ? WPATTN_OK : WPATTN_ECUDA;
}

int wpattn_rope(const void* x, void* out, int32_t B, int32_t N, int32_t H, int32_t head_dim,
                int64_t pos0, const int32_t* positions, double rope_base, void* cuda_stream) {
  if (B < 0 || N < 0 || H <= 0) return WPATTN_EINVAL;
  if (!(rope_base > 1.0) || std::isinf(rope_base)) return WPATTN_EINVAL;
  if (head_dim != 64 && head_dim != 128) return WPATTN_EUNSUPPORTED;
  if (B == 0 || N == 0) return WPATTN_OK;
  if (!x || !out || !aligned16(x) || !aligned16(out)) return WPATTN_EINVAL;
  if (positions && (reinterpret_cast<uintptr_t>(positions) & 3u) != 0) return WPATTN_EINVAL;
  if (!positions && (pos0 < 0 || pos0 > (int64_t(1) << 40))) return WPATTN_EINVAL;
  DeviceInfo* dev = nullptr;
  int rc;
  if ((rc = device_info(&dev)) != WPATTN_OK) return rc;
  return launch_rope(x, out, N, H, pos0, positions, nullptr, nullptr, 0, 0, 0, B, head_dim, rope_base,
                     dev->num_sms, static_cast<cudaStream_t>(cuda_stream));
}

int wpattn_rope_qk(const void* q, void* q_out, const void* k, void* k_out, int32_t B, int32_t Nq,
                   int32_t Nk, int32_t Hq, int32_t Hkv, int32_t head_dim, int64_t q_pos0, int64_t k_pos0,
                   double rope_base, void* cuda_stream) {
  if (B < 0 || Nq < 0 || Nk < 0 || Hq <= 0 || Hkv <= 0) return WPATTN_EINVAL;
  if (!(rope_base > 1.0) || std::isinf(rope_base)) return WPATTN_EINVAL;
  if (head_dim != 64 && head_dim != 128) return WPATTN_EUNSUPPORTED;
  if (q_pos0 < 0 || k_pos0 < 0 || q_pos0 > (int64_t(1) << 40) || k_pos0 > (int64_t(1) << 40))
    return WPATTN_EINVAL;
  if (B == 0 || (Nq == 0 && Nk == 0)) return WPATTN_OK;
  if (Nq > 0 && (!q || !q_out || !aligned16(q) || !aligned16(q_out))) return WPATTN_EINVAL;
  if (Nk > 0 && (!k || !k_out || !aligned16(k) || !aligned16(k_out))) return WPATTN_EINVAL;
  DeviceInfo* dev = nullptr;
  int rc;
  if ((rc = device_info(&dev)) != WPATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  if (Nq == 0)
    return launch_rope(k, k_out, Nk, Hkv, k_pos0, nullptr, nullptr, nullptr, 0, 0, 0, B, head_dim,
                       rope_base, dev->num_sms, st);
  return launch_rope(q, q_out, Nq, Hq, q_pos0, nullptr, Nk > 0 ? k : nullptr, k_out, Nk, Hkv, k_pos0, B,
                     head_dim, rope_base, dev->num_sms, st);
}

size_t wpattn_prefill_rope_workspace_size(int32_t B, int32_t Nq, int32_t Nk, int32_t Hq,
                                          int32_t Hkv, int32_t head_dim) {
  if (B < 0 || Nq < 0 || Nk < 0 || Hq <= 0 || Hkv <= 0 || head_dim <= 0) return 0;
  const size_t qb = static_cast<size_t>(B) * Nq * Hq * head_dim * 2;
  const size_t kb = static_cast<size_t>(B) * Nk * Hkv * head_dim * 2;
  return ((qb + 255) / 256) * 256 + kb;
}

int wpattn_prefill_rope(const wpattn_window* w, const void* q, const void* k, const void* v,
                        void* out, float* lse, int32_t B, int32_t Nq, int32_t Nk, int32_t Hq,
                        int32_t Hkv, int64_t q_pos0, int64_t k_pos0, float softmax_scale,
                        void* workspace, size_t workspace_bytes, void* cuda_stream) {
  WindowPlan plan;
  int rc = make_window_plan(w, &plan);
  if (rc != WPATTN_OK) return rc;
  if (B < 0 || Nq < 0 || Nk < 0 || Hq <= 0 || Hkv <= 0 || (Hq % Hkv) != 0) return WPATTN_EINVAL;
  if (plan.D != 64 && plan.D != 128) return WPATTN_EUNSUPPORTED;
  if (B == 0 || Nq == 0) return WPATTN_OK;
  const size_t need = wpattn_prefill_rope_workspace_size(B, Nq, Nk, Hq, Hkv, plan.D);
  if (!workspace || workspace_bytes < need) return WPATTN_EWORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return WPATTN_EINVAL;
  if (!q || !aligned16(q) || (Nk > 0 && (!k || !aligned16(k)))) return WPATTN_EINVAL;
  if (q_pos0 < 0 || k_pos0 < 0 || q_pos0 > (int64_t(1) << 40) || k_pos0 > (int64_t(1) << 40))
    return WPATTN_EINVAL;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* qr = ws;
  void* kr = ws + ((static_cast<size_t>(B) * Nq * Hq * plan.D * 2 + 255) / 256) * 256;
  // the rotations are a pre-pass: each key row is turned once, not once per
  // query block that reads it, and off the MUFU pipe the attention needs;
  // q and k go in one launch
  if ((rc = wpattn_rope_qk(q, qr, k, kr, B, Nq, Nk, Hq, Hkv, plan.D, q_pos0, k_pos0, w->rope_base,
                           cuda_stream)) != WPATTN_OK)
    return rc;
  return prefill_impl(w, qr, kr, v, out, lse, B, Nq, Nk, Hq, Hkv, q_pos0, k_pos0, softmax_scale,
                      nullptr, 0, cuda_stream);
}

size_t wpattn_decode_workspace_size(const wpattn_window* w, int32_t B, int32_t Hq, int32_t Hkv,
                                    int64_t max_kv_len) {
  WindowPlan plan;
  if (make_window_plan(w, &plan) != WPATTN_OK) return 0;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || (Hq % Hkv) != 0 || max_kv_len <= 0) return 0;
  return decode_workspace_bytes(B, Hq, plan.D, decode_max_splits(B, Hkv, max_kv_len));
}

}  // extern "C"

namespace {
// How the decode call finds its keys: the [B, Lmax, Hkv, D] cache (the
// default), pair-major K slabs, or page pools with a block table; and where
// they sit: at positions 0..kv_len-1 with the query last (the default), or at
// explicit positions.
struct DecodeLayout {
  bool pm = false;
  const int32_t* block_table = nullptr;   // device [B, max_pages]
  int max_pages = 0, page_size = 0, num_pages = 0;
  const int32_t* q_pos_host = nullptr;    // host [B]
  const int32_t* k_pos = nullptr;         // device [B, k_pos_stride]
  int64_t k_pos_stride = 0;
  bool rope_q = false;                    // q arrives before its RoPE rotation
  bool shard = false;                     // one shard of a longer cache: kv_len may be 0
};

int decode_impl(const wpattn_window* w, const void* q, const void* k_cache, const void* v_cache,
                const int32_t* kv_len_host, int64_t Lmax, int32_t B, int32_t Hq, int32_t Hkv,
                float softmax_scale, void* out, float* lse, void* workspace,
                size_t workspace_bytes, void* cuda_stream, const DecodeLayout& lay) {
  WindowPlan plan;
  int rc = make_window_plan(w, &plan);
  if (rc != WPATTN_OK) return rc;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || (Hq % Hkv) != 0 || Lmax <= 0) return WPATTN_EINVAL;
  if (!(softmax_scale == softmax_scale)) return WPATTN_EINVAL;
  if (!q || !k_cache || !v_cache || !kv_len_host || !out) return WPATTN_EINVAL;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
    return WPATTN_EINVAL;
  if (plan.D != 64 && plan.D != 128) return WPATTN_EUNSUPPORTED;
  const int G = Hq / Hkv;
  if (G > 16 || B > kDecodeMaxB || Lmax >= (int64_t(1) << 31)) return WPATTN_EUNSUPPORTED;
  for (int b = 0; b < B; ++b)
    if (kv_len_host[b] < (lay.shard ? 0 : 1) || kv_len_host[b] > Lmax) return WPATTN_EINVAL;
  if (lay.q_pos_host && !lay.shard)
    for (int b = 0; b < B; ++b)
      if (lay.q_pos_host[b] < 0 || lay.q_pos_host[b] == INT32_MAX) return WPATTN_EINVAL;
  if (lay.k_pos) {
    int32_t longest = 0;
    for (int b = 0; b < B; ++b) longest = std::max(longest, kv_len_host[b]);
    if (lay.k_pos_stride < longest || (reinterpret_cast<uintptr_t>(lay.k_pos) & 3u) != 0)
      return WPATTN_EINVAL;
  }
  DeviceInfo* dev = nullptr;
  if ((rc = device_info(&dev)) != WPATTN_OK) return rc;
  const int S = decode_splits(B, Hkv, Lmax, dev->decode_slots);
  const size_t need = decode_workspace_bytes(B, Hq, plan.D, S);
  if (!workspace || workspace_bytes < need) return WPATTN_EWORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return WPATTN_EINVAL;

  DecodeParams prm;
  std::memset(&prm, 0, sizeof prm);
  prm.q = static_cast<const uint16_t*>(q);
  prm.k = static_cast<const uint16_t*>(k_cache);
  prm.v = static_cast<const uint16_t*>(v_cache);
  prm.part = static_cast<float*>(workspace);
  prm.out = static_cast<uint16_t*>(out);
  prm.lse = lse;
  prm.Lmax = Lmax;
  prm.B = B; prm.Hq = Hq; prm.Hkv = Hkv; prm.G = G; prm.S = S;
  prm.hchunks = (G + 7) / 8;
  const int gc = (G + prm.hchunks - 1) / prm.hchunks;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(plan.D));
  prm.scale_log2 = scale * 1.44269504088896340736f;
  for (int p = 0; p < 64; ++p) prm.T[p] = plan.T[p] > INT32_MAX ? INT32_MAX : static_cast<int>(plan.T[p]);
  for (int b = 0; b < B; ++b) {
    prm.kv_len[b] = kv_len_host[b];
    prm.q_pos[b] = lay.q_pos_host ? lay.q_pos_host[b] : kv_len_host[b] - 1;
  }
  prm.block_table = lay.block_table;
  prm.max_pages = lay.max_pages;
  prm.page_size = lay.page_size;
  prm.num_pages = lay.num_pages;
  prm.k_pos = lay.k_pos;
  prm.k_pos_stride = lay.k_pos_stride;
  prm.rope_q = lay.rope_q ? 1 : 0;
  if (lay.rope_q) rope_thetas(w->rope_base, plan.D, prm.theta);
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  if (plan.D == 64) return launch_decode<64>(prm, gc, lay.pm, st);
  return launch_decode<128>(prm, gc, lay.pm, st);
}
}  // namespace

extern "C" {

int wpattn_decode(const wpattn_window* w, const void* q, const void* k_cache, const void* v_cache,
                  const int32_t* kv_len_host, int64_t Lmax, int32_t B, int32_t Hq, int32_t Hkv,
                  float softmax_scale, void* out, float* lse, void* workspace,
                  size_t workspace_bytes, void* cuda_stream) {
  return decode_impl(w, q, k_cache, v_cache, kv_len_host, Lmax, B, Hq, Hkv, softmax_scale, out, lse,
                     workspace, workspace_bytes, cuda_stream, DecodeLayout{});
}

int wpattn_decode_pairmajor(const wpattn_window* w, const void* q, const void* k_slabs,
                            const void* v_cache, const int32_t* kv_len_host, int64_t Lmax,
                            int32_t B, int32_t Hq, int32_t Hkv, float softmax_scale, void* out,
                            float* lse, void* workspace, size_t workspace_bytes,
                            void* cuda_stream) {
  DecodeLayout lay;
  lay.pm = true;
  return decode_impl(w, q, k_slabs, v_cache, kv_len_host, Lmax, B, Hq, Hkv, softmax_scale, out, lse,
                     workspace, workspace_bytes, cuda_stream, lay);
}

int wpattn_decode_positions(const wpattn_window* w, const void* q, const void* k_cache,
                            const void* v_cache, const int32_t* kv_len_host, int64_t Lmax,
                            const int32_t* q_pos_host, const int32_t* k_pos, int64_t k_pos_stride,
                            int32_t B, int32_t Hq, int32_t Hkv, float softmax_scale, void* out,
                            float* lse, void* workspace, size_t workspace_bytes,
                            void* cuda_stream) {
  if (!q_pos_host || !k_pos) return WPATTN_EINVAL;
  DecodeLayout lay;
  lay.q_pos_host = q_pos_host;
  lay.k_pos = k_pos;
  lay.k_pos_stride = k_pos_stride;
  return decode_impl(w, q, k_cache, v_cache, kv_len_host, Lmax, B, Hq, Hkv, softmax_scale, out, lse,
                     workspace, workspace_bytes, cuda_stream, lay);
}

int wpattn_decode_rope(const wpattn_window* w, const void* q, const void* k_cache,
                       const void* v_cache, const int32_t* kv_len_host, int64_t Lmax,
                       const int32_t* q_pos_host, const int32_t* k_pos, int64_t k_pos_stride,
                       int32_t B, int32_t Hq, int32_t Hkv, float softmax_scale, void* out,
                       float* lse, void* workspace, size_t workspace_bytes, void* cuda_stream) {
  if ((q_pos_host == nullptr) != (k_pos == nullptr)) return WPATTN_EINVAL;
  DecodeLayout lay;
  lay.rope_q = true;
  lay.q_pos_host = q_pos_host;
  lay.k_pos = k_pos;
  lay.k_pos_stride = k_pos_stride;
  return decode_impl(w, q, k_cache, v_cache, kv_len_host, Lmax, B, Hq, Hkv, softmax_scale, out, lse,
                     workspace, workspace_bytes, cuda_stream, lay);
}

int wpattn_decode_shard(const wpattn_window* w, const void* q, const void* k_shard,
                        const void* v_shard, const int32_t* kv_len_host, int64_t Lmax,
                        const int64_t* q_pos_host, const int64_t* k_pos0_host, int32_t B,
                        int32_t Hq, int32_t Hkv, float softmax_scale, void* out, float* lse,
                        void* workspace, size_t workspace_bytes, void* cuda_stream) {
  if (!q_pos_host || !k_pos0_host || !lse || !kv_len_host || B <= 0 || B > kDecodeMaxB)
    return WPATTN_EINVAL;
  // the kernel measures distances from the shard's first key: the query sits
  // at q_pos - k_pos0, the shard's key j at j, every one of them before it
  int32_t rel[kDecodeMaxB];
  for (int b = 0; b < B; ++b) {
    const int64_t r = q_pos_host[b] - k_pos0_host[b];
    if (q_pos_host[b] < 0 || k_pos0_host[b] < 0 || r >= INT32_MAX) return WPATTN_EINVAL;
    if (kv_len_host[b] > 0 && r < static_cast<int64_t>(kv_len_host[b]) - 1) return WPATTN_EINVAL;
    rel[b] = kv_len_host[b] > 0 ? static_cast<int32_t>(r) : 0;
  }
  DecodeLayout lay;
  lay.shard = true;
  lay.q_pos_host = rel;
  return decode_impl(w, q, k_shard, v_shard, kv_len_host, Lmax, B, Hq, Hkv, softmax_scale, out, lse,
                     workspace, workspace_bytes, cuda_stream, lay);
}

int wpattn_merge_lse(const void* outs, const float* lses, int32_t R, int64_t rows, int32_t head_dim,
                     void* out, float* lse, void* cuda_stream) {
  if (R <= 0 || rows < 0) return WPATTN_EINVAL;
  if (head_dim != 64 && head_dim != 128) return WPATTN_EUNSUPPORTED;
  if (rows == 0) return WPATTN_OK;
  if (!outs || !lses || !out || rows > 0x7FFFFFFFLL) return WPATTN_EINVAL;
  DeviceInfo* dev = nullptr;
  int rc;
  if ((rc = device_info(&dev)) != WPATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  if (head_dim == 64)
    merge_lse_kernel<64><<<static_cast<unsigned>(rows), 64, 0, st>>>(
        static_cast<const uint16_t*>(outs), lses, R, rows, static_cast<uint16_t*>(out), lse);
  else
    merge_lse_kernel<128><<<static_cast<unsigned>(rows), 128, 0, st>>>(
        static_cast<const uint16_t*>(outs), lses, R, rows, static_cast<uint16_t*>(out), lse);
  return cudaGetLastError() == cudaSuccess ? WPATTN_OK : WPATTN_ECUDA;
}

int wpattn_decode_paged(const wpattn_window* w, const void* q, const void* k_pages,
                        const void* v_pages, int32_t num_pages, int32_t page_size,
                        const int32_t* block_table, int32_t max_pages_per_seq,
                        const int32_t* kv_len_host, const int32_t* q_pos_host,
                        const int32_t* k_pos, int64_t k_pos_stride, int32_t B, int32_t Hq,
                        int32_t Hkv, float softmax_scale, void* out, float* lse, void* workspace,
                        size_t workspace_bytes, void* cuda_stream) {
  if (!block_table || num_pages <= 0 || max_pages_per_seq <= 0) return WPATTN_EINVAL;
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) != 0) return WPATTN_EINVAL;
  // a 32-key block is one page, a part of one page, or a whole number of pages
  if (!(page_size == 8 || page_size == 16 || (page_size > 0 && page_size % 32 == 0)))
    return WPATTN_EUNSUPPORTED;
  if ((q_pos_host == nullptr) != (k_pos == nullptr)) return WPATTN_EINVAL;
  const int64_t cap = static_cast<int64_t>(max_pages_per_seq) * page_size;
  if (static_cast<int64_t>(num_pages) * page_size >= (int64_t(1) << 40)) return WPATTN_EUNSUPPORTED;
  DecodeLayout lay;
  lay.block_table = block_table;
  lay.max_pages = max_pages_per_seq;
  lay.page_size = page_size;
  lay.num_pages = num_pages;
  lay.q_pos_host = q_pos_host;
  lay.k_pos = k_pos;
  lay.k_pos_stride = k_pos_stride;
  return decode_impl(w, q, k_pages, v_pages, kv_len_host, cap, B, Hq, Hkv, softmax_scale, out, lse,
                     workspace, workspace_bytes, cuda_stream, lay);
}

int wpattn_kcache_to_pairmajor(const void* k_cache, void* k_slabs, int64_t Lmax, int32_t B,
                               int32_t Hkv, int32_t head_dim, void* cuda_stream) {
  if (!k_cache || !k_slabs || Lmax <= 0 || B <= 0 || Hkv <= 0) return WPATTN_EINVAL;
  if (!aligned16(k_cache) || !aligned16(k_slabs)) return WPATTN_EINVAL;
  if (head_dim != 64 && head_dim != 128) return WPATTN_EUNSUPPORTED;
  if (Lmax >= (int64_t(1) << 31)) return WPATTN_EUNSUPPORTED;
  DeviceInfo* dev = nullptr;
  int rc;
  if ((rc = device_info(&dev)) != WPATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  const uint64_t n = static_cast<uint64_t>(B) * Hkv * (head_dim / 16) * static_cast<uint64_t>(Lmax);
  const uint64_t blocks = (n + 255) / 256;
  if (blocks > 0x7FFFFFFFull) return WPATTN_EUNSUPPORTED;
  if (head_dim == 64)
    kcache_to_pairmajor_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        static_cast<const uint16_t*>(k_cache), static_cast<uint16_t*>(k_slabs), Lmax, B, Hkv);
  else
    kcache_to_pairmajor_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        static_cast<const uint16_t*>(k_cache), static_cast<uint16_t*>(k_slabs), Lmax, B, Hkv);
  return cudaGetLastError() == cudaSuccess ? WPATTN_OK : WPATTN_ECUDA;
}

size_t wpattn_decode_noalloc_max_bytes(void) { return kDecodeStaticScratchBytes; }

int wpattn_decode_noalloc(const wpattn_window* w, const void* q, const void* k_cache,
                          const void* v_cache, const int32_t* kv_len_host, int64_t Lmax, int32_t B,
                          int32_t Hq, int32_t Hkv, float softmax_scale, void* out, float* lse,
                          void* cuda_stream) {
  WindowPlan plan;
  int rc = make_window_plan(w, &plan);
  if (rc != WPATTN_OK) return rc;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || (Hq % Hkv) != 0 || Lmax <= 0) return WPATTN_EINVAL;
  DeviceInfo* dev = nullptr;
  if ((rc = device_info(&dev)) != WPATTN_OK) return rc;
  // scratch this problem needs under the current device's split plan
  const int S = decode_splits(B, Hkv, Lmax, dev->decode_slots);
  if (decode_workspace_bytes(B, Hq, plan.D, S) > kDecodeStaticScratchBytes) return WPATTN_EWORKSPACE;
  {
    // once per device, with that device current: the array's device address
    // (host code cannot use the symbol itself as a device pointer)
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!dev->static_scratch) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_decode_static_scratch) != cudaSuccess || !ptr)
        return WPATTN_ECUDA;
      dev->static_scratch = ptr;
    }
  }
  return wpattn_decode(w, q, k_cache, v_cache, kv_len_host, Lmax, B, Hq, Hkv, softmax_scale, out,
                       lse, dev->static_scratch, kDecodeStaticScratchBytes, cuda_stream);
}

int wpattn_selftest_wait_timeout(void* cuda_stream) {
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc != WPATTN_OK) return rc;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(cuda_stream)>>>();
  return cudaGetLastError() == cudaSuccess ? WPATTN_OK : WPATTN_ECUDA;
}

int wpattn_device_status(void* cuda_stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess)
    return WPATTN_ECUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof v) != cudaSuccess) return WPATTN_ECUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof zero) != cudaSuccess) return WPATTN_ECUDA;
  }
  return v == 0 ? WPATTN_OK : v;
}

}  // extern "C"
