// C-ABI library: argument validation, dynamic factor, workspace layout, TMA
// descriptors and kernel dispatch. Built as one translation unit with the kernels so
// that the device status word is a single object.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>

#include "../../include/bifocal.h"
#include "common.cuh"
#include "decode.cuh"
#include "prefill_mma.cuh"
#include "prefill_tc.cuh"
#include "prefill_tc2.cuh"
#include "rope_prepass.cuh"

namespace {

using bf16 = __nv_bfloat16;

constexpr int kMaxSplits = 320;  // split-KV partials reserved in the decode workspace

// Test-only fault injection (bifocal_test_set_fault), passed to the kernels as arguments: one
// more than the fill of the prefill producer / the stage of the decode producer that CTA 0 never
// issues; 0 = off (so an argument block cleared to zero never skips anything).
int g_test_skip_fill = 0;
int g_test_skip_stage = 0;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct Rope {
  double omega[64];
  double omega_long[64];
  double omega_corr[64];
};

// omega_k = theta^(-2k/D) in fp64 on the host; long-range forms for factor G.
Rope make_rope(double theta, int D, int G) {
  // A decode loop asks for the same tables every step: keep the last set per thread (64 pow
  // calls are a few microseconds of host time, as much as a short decode step takes on the GPU).
  thread_local double last_theta = 0.0;
  thread_local int last_D = 0, last_G = 0;
  thread_local Rope last;
  if (theta == last_theta && D == last_D && G == last_G) return last;
  Rope r;
  std::memset(&r, 0, sizeof(r));
  for (int k = 0; k < D / 2; ++k) {
    const double om = std::pow(theta, -2.0 * k / D);
    r.omega[k] = om;
    r.omega_long[k] = om / G;
    r.omega_corr[k] = om / G - om;
  }
  last = r;
  last_theta = theta;
  last_D = D;
  last_G = G;
  return r;
}

int factor(int64_t L, int w) { return L <= w ? 1 : static_cast<int>((L + w - 1) / w); }

bf_status_t check_params(const bf_params_t* p, bool need_window) {
  if (!p) return BF_ERR_INVALID;
  if (p->hq < 1 || p->hkv < 1 || p->hq % p->hkv) return BF_ERR_INVALID;
  if (p->head_dim != 64 && p->head_dim != 128) return BF_ERR_UNSUPPORTED;
  if (!(p->rope_theta > 1.0) || !std::isfinite(p->rope_theta)) return BF_ERR_INVALID;
  if (!(p->softmax_scale >= 0.f) || !std::isfinite(p->softmax_scale)) return BF_ERR_INVALID;
  if (need_window) {
    if (p->w0 < 0 || p->w_pretrained < 1) return BF_ERR_INVALID;
    if (p->mode != BF_MODE_FREQ_INTERP && p->mode != BF_MODE_POS_ALIAS) return BF_ERR_INVALID;
  }
  return BF_OK;
}

float scale_log2(const bf_params_t* p) {
  const double s = p->softmax_scale > 0.f ? p->softmax_scale : 1.0 / std::sqrt(static_cast<double>(p->head_dim));
  return static_cast<float>(s * 1.4426950408889634073599246810019);
}

int sm_count() {
  static std::atomic<int> cached[64];  // per device ordinal, 0 = not asked yet
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64 && (n = cached[dev].load(std::memory_order_relaxed)) > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

// ------------------------------------------------------------------ TMA descriptors
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// Cache [cap, hkv, D] bf16 viewed as (d_lo = 64, d_hi = D/64, head, key) with a box of
// (64, 1, 1, kb) and the 128-byte swizzle: one 128-byte row per key.
bool make_cache_map(CUtensorMap* map, const void* base, int cap, int hkv, int D, int kb) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(D / 64), static_cast<cuuint64_t>(hkv), static_cast<cuuint64_t>(cap)};
  cuuint64_t strides[3] = {128, static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(hkv) * D * 2};
  cuuint32_t box[4] = {64, 1, 1, static_cast<cuuint32_t>(kb)};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Launch with programmatic stream serialisation: the kernel may start while the previous
// kernel on the stream is still running; it synchronises with griddepcontrol.wait.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Rotated key forms [rows = b*hkv][L][128] fp16, box (64, 128, 1), 128B swizzle.
bool make_k_map(CUtensorMap* map, const void* base, int L, int rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(L) * 256};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// V [b][L][hkv][128] bf16, box (64, 1, box_rows, 1), 128B swizzle: one 128-byte row per key.
bool make_v_map(CUtensorMap* map, const void* base, int L, int hkv, int batch, int box_rows = 128) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {128, static_cast<cuuint64_t>(hkv), static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[3] = {256, static_cast<cuuint64_t>(hkv) * 256, static_cast<cuuint64_t>(L) * hkv * 256};
  cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ prefill
struct PrefillLayout {
  size_t qo, ql, ko, kl, vb, total;
};

bool tc2_path(const bf_params_t* p);

// The fused-load path: RoPE and the correction rotation inside the ping-pong kernel's tile
// loads (bf16 inputs, D = 128, even GQA group), selected by BF_FLAG_FUSED_ROPE.
bool fused_path(const bf_params_t* p, int dtype) {
  return (p->flags & BF_FLAG_FUSED_ROPE) && dtype == BF_DTYPE_BF16 && tc2_path(p);
}

PrefillLayout prefill_layout(int dtype, int batch, int L, const bf_params_t* p) {
  PrefillLayout w{};
  if (fused_path(p, dtype)) return w;  // nothing to stage: every operand is formed in the kernel
  const size_t qbytes = align256(static_cast<size_t>(batch) * L * p->hq * p->head_dim * 2);
  const size_t kbytes = align256(static_cast<size_t>(batch) * L * p->hkv * p->head_dim * 2);
  w.qo = 0;
  w.ql = w.qo + qbytes;
  w.ko = w.ql + qbytes;
  w.kl = w.ko + kbytes;
  w.vb = w.kl + kbytes;
  w.total = w.vb + (dtype == BF_DTYPE_FP32 ? kbytes : 0);
  return w;
}

template <int D, bool BIF>
cudaError_t launch_attn_mma(const bf::AttnArgs& a, int batch, cudaStream_t st) {
  constexpr int smem = bf::attn_mma_smem_bytes<D, BIF>();
  cudaError_t e = cudaFuncSetAttribute(bf::attn_mma_kernel<D, BIF>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.L + bf::mma_cfg::BM - 1) / bf::mma_cfg::BM, a.hq, batch);
  bf::attn_mma_kernel<D, BIF><<<grid, bf::mma_cfg::WARPS * 32, smem, st>>>(a);
  return cudaGetLastError();
}

// The tcgen05 ping-pong kernel (two heads of one GQA group per CTA) takes D = 128 and an even group.
bool tc2_path(const bf_params_t* p) {
  const int g = p->hq / p->hkv;
  return p->head_dim == 128 && !(p->flags & BF_FLAG_MMA_SYNC) && p->hq % 2 == 0 && g % 2 == 0;
}

// What a prefill call resolves before any launch (shared by the one-call form and the
// two steps, so both make the same choice).
struct PrefillPlan {
  int D, G;
  bool bif;  // two-branch kernel (else every pair is local: the plain kernel gives the same result)
  int kind;  // tcgen05 ping-pong kernel: KIND_PLAIN, KIND_BIFOCAL or KIND_WINDOW
  bool fused;  // RoPE in the kernel's tile loads (no rotated copies in the workspace)
  PrefillLayout lay;
  Rope rope;
};

bf_status_t plan_prefill(bool bifocal_api, int32_t dtype, int32_t batch, int32_t L, const bf_params_t* p,
                         void* workspace, size_t ws_bytes, PrefillPlan* plan) {
  bf_status_t s = check_params(p, bifocal_api);
  if (s != BF_OK) return s;
  if (batch < 1 || L < 1) return BF_ERR_INVALID;
  if (dtype != BF_DTYPE_BF16 && dtype != BF_DTYPE_FP32) return BF_ERR_UNSUPPORTED;
  const bool window = bifocal_api && (p->flags & BF_FLAG_WINDOW);
  if (window && p->w0 < 1) return BF_ERR_INVALID;
  if (window && !tc2_path(p)) return BF_ERR_UNSUPPORTED;
  plan->lay = prefill_layout(dtype, batch, L, p);
  if (plan->lay.total > 0 && (!workspace || !aligned(workspace, 256) || ws_bytes < plan->lay.total))
    return BF_ERR_WORKSPACE;
  plan->fused = fused_path(p, dtype);
  plan->D = p->head_dim;
  plan->G = bifocal_api ? factor(L, p->w_pretrained) : 1;
  plan->bif = !window && bifocal_api && ((p->flags & BF_FLAG_FORCE_BIFOCAL) || (plan->G > 1 && p->w0 < L));
  plan->kind = window ? (p->w0 < L ? bf::tc2::KIND_WINDOW : bf::tc2::KIND_PLAIN) : (plan->bif ? bf::tc2::KIND_BIFOCAL : bf::tc2::KIND_PLAIN);
  plan->rope = make_rope(p->rope_theta, plan->D, plan->G);
  return BF_OK;
}

bf_status_t prefill_rope_impl(bool bifocal_api, const void* q, const void* k, const void* v, int32_t dtype,
                              int32_t batch, int32_t L, const bf_params_t* p, void* kcache_out, void* vcache_out,
                              void* workspace, size_t ws_bytes, void* stream, const void* q_norm_w = nullptr,
                              const void* k_norm_w = nullptr, float norm_eps = 0.f) {
  PrefillPlan plan;
  bf_status_t s = check_params(p, bifocal_api);
  if (s != BF_OK) return s;
  if (!q || !k || !v) return BF_ERR_INVALID;
  const size_t align_in = dtype == BF_DTYPE_FP32 ? 32 : 16;
  if (!aligned(q, align_in) || !aligned(k, align_in) || !aligned(v, align_in)) return BF_ERR_INVALID;
  if ((kcache_out && !aligned(kcache_out, 16)) || (vcache_out && !aligned(vcache_out, 16))) return BF_ERR_INVALID;
  s = plan_prefill(bifocal_api, dtype, batch, L, p, workspace, ws_bytes, &plan);
  if (s != BF_OK) return s;
  const int D = plan.D;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  bf::PrepassArgs pa{};
  pa.q = q;
  pa.k = k;
  pa.v = v;
  pa.batch = batch;
  pa.L = L;
  pa.pos0 = 0;
  pa.Lk = L;
  pa.Lc = L;
  pa.hq = p->hq;
  pa.hkv = p->hkv;
  pa.G = plan.G;
  pa.mode = bifocal_api ? p->mode : 0;
  pa.need_long = plan.bif ? 1 : 0;
  pa.Qo = reinterpret_cast<__half*>(ws + plan.lay.qo);
  pa.Ql = reinterpret_cast<__half*>(ws + plan.lay.ql);
  pa.Ko = reinterpret_cast<__half*>(ws + plan.lay.ko);
  pa.Kl = reinterpret_cast<__half*>(ws + plan.lay.kl);
  pa.Vb = dtype == BF_DTYPE_FP32 ? reinterpret_cast<bf16*>(ws + plan.lay.vb) : nullptr;
  pa.kcache = static_cast<bf16*>(kcache_out);
  pa.vcache = static_cast<bf16*>(vcache_out);
  std::memcpy(pa.omega, plan.rope.omega, sizeof(pa.omega));
  std::memcpy(pa.omega_long, plan.rope.omega_long, sizeof(pa.omega_long));
  pa.q_norm_w = q_norm_w;
  pa.k_norm_w = k_norm_w;
  pa.norm_eps = norm_eps;
  if (plan.fused) {
    // the attention kernel forms every operand itself: this step only writes the cache rows asked for
    if (!kcache_out && !vcache_out) return BF_OK;
    pa.keys_only = 1;
    pa.need_long = 0;
    pa.Qo = pa.Ql = pa.Ko = pa.Kl = nullptr;
  }
  const long long rows = static_cast<long long>(batch) * L;
  const dim3 pgrid(static_cast<unsigned>((rows + 7) / 8));
  if (dtype == BF_DTYPE_BF16) {
    if (D == 128)
      bf::rope_prepass_kernel<bf16, 128><<<pgrid, 256, 0, st>>>(pa);
    else
      bf::rope_prepass_kernel<bf16, 64><<<pgrid, 256, 0, st>>>(pa);
  } else {
    if (D == 128)
      bf::rope_prepass_kernel<float, 128><<<pgrid, 256, 0, st>>>(pa);
    else
      bf::rope_prepass_kernel<float, 64><<<pgrid, 256, 0, st>>>(pa);
  }
  return cudaGetLastError() == cudaSuccess ? BF_OK : BF_ERR_CUDA;
}

template <bool FUSED>
cudaError_t launch_tc2_t(int kind, const bf::Tc2Args& ta, long long n_cta, cudaStream_t st) {
  constexpr int smem = bf::attn_tc2_smem_bytes(FUSED);
  auto kern = kind == bf::tc2::KIND_BIFOCAL  ? bf::attn_tc2_kernel<bf::tc2::KIND_BIFOCAL, FUSED>
              : kind == bf::tc2::KIND_WINDOW ? bf::attn_tc2_kernel<bf::tc2::KIND_WINDOW, FUSED>
                                             : bf::attn_tc2_kernel<bf::tc2::KIND_PLAIN, FUSED>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<static_cast<unsigned>(n_cta), bf::tc2::NTHREADS2, smem, st>>>(ta);
  return cudaGetLastError();
}

cudaError_t launch_tc2(int kind, bool fused, const bf::Tc2Args& ta, long long n_cta, cudaStream_t st) {
  return fused ? launch_tc2_t<true>(kind, ta, n_cta, st) : launch_tc2_t<false>(kind, ta, n_cta, st);
}

// The fused ping-pong attention over raw bf16 q [batch, Lq, hq, 128] (rows at absolute positions
// q_off..) and a key source [batch, L, hkv, 128] (raw k, or the cache of original-RoPE keys)
// with V [batch, L, hkv, 128].
bf_status_t fused_attention(int kind, const void* q, const void* ksrc, bool cache, const void* v, int batch, int L,
                            int q_off, int Lq, int G, const bf_params_t* p, const Rope& rope, void* out, float* lse,
                            cudaStream_t st) {
  bf::Tc2Args ta;
  std::memset(&ta, 0, sizeof(ta));
  if (!make_v_map(&ta.v_map, v, L, p->hkv, batch) || !make_v_map(&ta.qo_map, q, Lq, p->hq, batch) ||
      !make_v_map(&ta.ko_map, ksrc, L, p->hkv, batch))
    return BF_ERR_CUDA;
  ta.out = static_cast<bf16*>(out);
  ta.lse = lse;
  ta.L = L;
  ta.hq = p->hq;
  ta.hkv = p->hkv;
  ta.batch = batch;
  ta.w0 = kind != bf::tc2::KIND_PLAIN ? p->w0 : L;
  ta.q_off = q_off;
  ta.Lq = Lq;
  ta.scale_log2 = scale_log2(p);
  ta.test_skip_fill = g_test_skip_fill;
  ta.src.cache = cache ? 1 : 0;
  ta.src.mode = p->mode;
  ta.src.G = G;
  std::memcpy(ta.src.omega, rope.omega, sizeof(ta.src.omega));
  const long long n_cta = static_cast<long long>((Lq + bf::tc::BM - 1) / bf::tc::BM) * (p->hq / 2) * batch;
  if (n_cta > 0x7fffffffLL) return BF_ERR_UNSUPPORTED;
  return launch_tc2(kind, true, ta, n_cta, st) == cudaSuccess ? BF_OK : BF_ERR_CUDA;
}

bf_status_t prefill_attention_impl(bool bifocal_api, const void* v, int32_t dtype, int32_t batch, int32_t L,
                                   const bf_params_t* p, void* out, float* lse, void* workspace, size_t ws_bytes,
                                   void* stream) {
  PrefillPlan plan;
  bf_status_t s = check_params(p, bifocal_api);
  if (s != BF_OK) return s;
  if (!v || !out) return BF_ERR_INVALID;
  if (!aligned(v, dtype == BF_DTYPE_FP32 ? 32 : 16) || !aligned(out, 16) || (lse && !aligned(lse, 4)))
    return BF_ERR_INVALID;
  s = plan_prefill(bifocal_api, dtype, batch, L, p, workspace, ws_bytes, &plan);
  if (s != BF_OK) return s;
  if (plan.fused) return BF_ERR_UNSUPPORTED;  // the fused kernel reads q and k itself: use the one-call form
  const int D = plan.D;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  bf::AttnArgs aa{};
  aa.Qo = reinterpret_cast<const __half*>(ws + plan.lay.qo);
  aa.Ql = reinterpret_cast<const __half*>(ws + plan.lay.ql);
  aa.Ko = reinterpret_cast<const __half*>(ws + plan.lay.ko);
  aa.Kl = reinterpret_cast<const __half*>(ws + plan.lay.kl);
  aa.V = dtype == BF_DTYPE_FP32 ? reinterpret_cast<const bf16*>(ws + plan.lay.vb) : static_cast<const bf16*>(v);
  aa.v_row_stride = static_cast<long long>(p->hkv) * D;
  aa.v_batch_stride = static_cast<long long>(L) * p->hkv * D;
  aa.out = static_cast<bf16*>(out);
  aa.lse = lse;
  aa.L = L;
  aa.hq = p->hq;
  aa.hkv = p->hkv;
  aa.w0 = plan.kind != bf::tc2::KIND_PLAIN ? p->w0 : L;
  aa.scale_log2 = scale_log2(p);
  cudaError_t e;
  if (tc2_path(p)) {
    // tcgen05 ping-pong path: two heads of one GQA group per CTA
    bf::Tc2Args ta;
    std::memset(&ta, 0, sizeof(ta));
    if (!make_k_map(&ta.qo_map, aa.Qo, L, batch * p->hq) || !make_k_map(&ta.ql_map, aa.Ql, L, batch * p->hq) ||
        !make_k_map(&ta.ko_map, aa.Ko, L, batch * p->hkv) || !make_k_map(&ta.kl_map, aa.Kl, L, batch * p->hkv) ||
        !make_v_map(&ta.v_map, aa.V, L, p->hkv, batch))
      return BF_ERR_CUDA;
    ta.out = aa.out;
    ta.lse = aa.lse;
    ta.L = L;
    ta.hq = p->hq;
    ta.hkv = p->hkv;
    ta.batch = batch;
    ta.w0 = aa.w0;
    ta.q_off = 0;
    ta.Lq = L;
    ta.scale_log2 = aa.scale_log2;
    ta.test_skip_fill = g_test_skip_fill;
    constexpr int smem = bf::attn_tc2_smem_bytes();
    const long long n_cta = static_cast<long long>((L + bf::tc::BM - 1) / bf::tc::BM) * (p->hq / 2) * batch;
    if (n_cta > 0x7fffffffLL) return BF_ERR_UNSUPPORTED;
    auto kern = plan.kind == bf::tc2::KIND_BIFOCAL  ? bf::attn_tc2_kernel<bf::tc2::KIND_BIFOCAL, false>
                : plan.kind == bf::tc2::KIND_WINDOW ? bf::attn_tc2_kernel<bf::tc2::KIND_WINDOW, false>
                                               : bf::attn_tc2_kernel<bf::tc2::KIND_PLAIN, false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) {
      kern<<<static_cast<unsigned>(n_cta), bf::tc2::NTHREADS2, smem, st>>>(ta);
      e = cudaGetLastError();
    }
  } else if (D == 128 && !(p->flags & BF_FLAG_MMA_SYNC)) {
    // tcgen05 single-tile path (odd GQA groups)
    bf::TcArgs ta;
    std::memset(&ta, 0, sizeof(ta));
    if (!make_k_map(&ta.ko_map, aa.Ko, L, batch * p->hkv) || !make_k_map(&ta.kl_map, aa.Kl, L, batch * p->hkv) ||
        !make_v_map(&ta.v_map, aa.V, L, p->hkv, batch))
      return BF_ERR_CUDA;
    ta.Qo = aa.Qo;
    ta.Ql = aa.Ql;
    ta.out = aa.out;
    ta.lse = aa.lse;
    ta.L = L;
    ta.hq = p->hq;
    ta.hkv = p->hkv;
    ta.batch = batch;
    ta.w0 = aa.w0;
    ta.scale_log2 = aa.scale_log2;
    constexpr int smem = bf::attn_tc_smem_bytes();
    const long long n_cta = static_cast<long long>((L + bf::tc::BM - 1) / bf::tc::BM) * p->hq * batch;
    if (n_cta > 0x7fffffffLL) return BF_ERR_UNSUPPORTED;
    auto kern = plan.bif ? bf::attn_tc_kernel<true> : bf::attn_tc_kernel<false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) {
      kern<<<static_cast<unsigned>(n_cta), bf::tc::NTHREADS, smem, st>>>(ta);
      e = cudaGetLastError();
    }
  } else if (D == 128) {
    e = plan.bif ? launch_attn_mma<128, true>(aa, batch, st) : launch_attn_mma<128, false>(aa, batch, st);
  } else {
    e = plan.bif ? launch_attn_mma<64, true>(aa, batch, st) : launch_attn_mma<64, false>(aa, batch, st);
  }
  return e == cudaSuccess ? BF_OK : BF_ERR_CUDA;
}

// ------------------------------------------------------------------ chunked prefill
struct ChunkLayout {
  size_t qo, ql, ko, kl, total;
};

ChunkLayout chunk_layout(int P0, int C, const bf_params_t* p, int dtype) {
  ChunkLayout w{};
  if (fused_path(p, dtype)) return w;  // cached keys are re-phased in the kernel's tile loads
  const size_t qbytes = align256(static_cast<size_t>(C) * p->hq * p->head_dim * 2);
  const size_t kbytes = align256((static_cast<size_t>(P0) + C) * p->hkv * p->head_dim * 2);
  w.qo = 0;
  w.ql = w.qo + qbytes;
  w.ko = w.ql + qbytes;
  w.kl = w.ko + kbytes;
  w.total = w.kl + kbytes;
  return w;
}

bf_status_t chunk_impl(const void* q, const void* k, const void* v, int32_t dtype, int32_t P0, int32_t C,
                       const bf_params_t* p, void* kcache, void* vcache, int32_t cap, void* out, float* lse,
                       void* workspace, size_t ws_bytes, void* stream) {
  // validate everything before the first launch
  bf_status_t s = check_params(p, true);
  if (s != BF_OK) return s;
  if (!q || !k || !v || !out || !kcache || !vcache) return BF_ERR_INVALID;
  if (P0 < 0 || C < 1 || cap < 1 || static_cast<int64_t>(P0) + C > cap) return BF_ERR_INVALID;
  if (dtype != BF_DTYPE_BF16 && dtype != BF_DTYPE_FP32) return BF_ERR_UNSUPPORTED;
  const int D = p->head_dim, g = p->hq / p->hkv;
  if (D != 128 || p->hq % 2 || g % 2 || (p->flags & BF_FLAG_MMA_SYNC)) return BF_ERR_UNSUPPORTED;
  const size_t align_in = dtype == BF_DTYPE_FP32 ? 32 : 16;
  if (!aligned(q, align_in) || !aligned(k, align_in) || !aligned(v, align_in) || !aligned(kcache, 16) ||
      !aligned(vcache, 16) || !aligned(out, 16) || (lse && !aligned(lse, 4)))
    return BF_ERR_INVALID;
  const int L = P0 + C;
  const bool window = (p->flags & BF_FLAG_WINDOW) != 0;
  if (window && p->w0 < 1) return BF_ERR_INVALID;
  const ChunkLayout lay = chunk_layout(P0, C, p, dtype);
  if (lay.total > 0 && (!workspace || !aligned(workspace, 256) || ws_bytes < lay.total)) return BF_ERR_WORKSPACE;
  const int G = factor(L, p->w_pretrained);
  const bool bif = !window && ((p->flags & BF_FLAG_FORCE_BIFOCAL) || (G > 1 && p->w0 < L));
  const int kind = window ? (p->w0 < L ? bf::tc2::KIND_WINDOW : bf::tc2::KIND_PLAIN) : (bif ? bf::tc2::KIND_BIFOCAL : bf::tc2::KIND_PLAIN);
  const Rope rope = make_rope(p->rope_theta, D, G);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (fused_path(p, dtype)) {
    // 1. the chunk's keys (original RoPE, bf16) and values into cache rows P0 ..
    bf::PrepassArgs pa{};
    pa.q = q;
    pa.k = k;
    pa.v = v;
    pa.batch = 1;
    pa.L = C;
    pa.pos0 = P0;
    pa.Lk = L;
    pa.Lc = cap;
    pa.hq = p->hq;
    pa.hkv = p->hkv;
    pa.G = G;
    pa.mode = p->mode;
    pa.keys_only = 1;
    pa.kcache = static_cast<bf16*>(kcache);
    pa.vcache = static_cast<bf16*>(vcache);
    std::memcpy(pa.omega, rope.omega, sizeof(pa.omega));
    bf::rope_prepass_kernel<bf16, 128><<<static_cast<unsigned>((C + 7) / 8), 256, 0, st>>>(pa);
    if (cudaGetLastError() != cudaSuccess) return BF_ERR_CUDA;
    // 2. the chunk's queries over all L cached keys, read as stored and re-phased in the tile loads
    return fused_attention(kind, q, kcache, true, vcache, 1, L, P0, C, G, p, rope, out, lse, st);
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  __half* Qo = reinterpret_cast<__half*>(ws + lay.qo);
  __half* Ql = reinterpret_cast<__half*>(ws + lay.ql);
  __half* Ko = reinterpret_cast<__half*>(ws + lay.ko);
  __half* Kl = reinterpret_cast<__half*>(ws + lay.kl);

  // 1. cached keys -> Ko (fp16 copy) and Kl (correction rotation). A window reads only the
  //    cached keys within w0 of the chunk, from the start of their key tile on.
  const int j_begin = kind == bf::tc2::KIND_WINDOW ? std::max(0, (P0 + 1 - p->w0) / bf::tc::BN * bf::tc::BN) : 0;
  if (P0 > j_begin) {
    bf::RephaseArgs ra{};
    ra.kcache = static_cast<const bf16*>(kcache);
    ra.P0 = P0;
    ra.hkv = p->hkv;
    ra.Lk = L;
    ra.j_begin = j_begin;
    ra.G = G;
    ra.mode = p->mode;
    ra.need_long = bif ? 1 : 0;
    ra.Ko = Ko;
    ra.Kl = Kl;
    std::memcpy(ra.omega, rope.omega, sizeof(ra.omega));
    std::memcpy(ra.omega_corr, rope.omega_corr, sizeof(ra.omega_corr));
    bf::cache_rephase_kernel<128><<<static_cast<unsigned>((P0 - j_begin + 7) / 8), 256, 0, st>>>(ra);
    if (cudaGetLastError() != cudaSuccess) return BF_ERR_CUDA;
  }
  // 2. the chunk: RoPE forms of q and k at positions P0.., key rows P0.., cache rows P0..
  bf::PrepassArgs pa{};
  pa.q = q;
  pa.k = k;
  pa.v = v;
  pa.batch = 1;
  pa.L = C;
  pa.pos0 = P0;
  pa.Lk = L;
  pa.Lc = cap;
  pa.hq = p->hq;
  pa.hkv = p->hkv;
  pa.G = G;
  pa.mode = p->mode;
  pa.need_long = bif ? 1 : 0;
  pa.Qo = Qo;
  pa.Ql = Ql;
  pa.Ko = Ko;
  pa.Kl = Kl;
  pa.Vb = nullptr;
  pa.kcache = static_cast<bf16*>(kcache);
  pa.vcache = static_cast<bf16*>(vcache);
  std::memcpy(pa.omega, rope.omega, sizeof(pa.omega));
  std::memcpy(pa.omega_long, rope.omega_long, sizeof(pa.omega_long));
  const dim3 pgrid(static_cast<unsigned>((C + 7) / 8));
  if (dtype == BF_DTYPE_BF16)
    bf::rope_prepass_kernel<bf16, 128><<<pgrid, 256, 0, st>>>(pa);
  else
    bf::rope_prepass_kernel<float, 128><<<pgrid, 256, 0, st>>>(pa);
  if (cudaGetLastError() != cudaSuccess) return BF_ERR_CUDA;
  // 3. attention of the C query rows (absolute positions P0..) over keys 0..L-1; V is the cache
  bf::Tc2Args ta;
  std::memset(&ta, 0, sizeof(ta));
  if (!make_k_map(&ta.qo_map, Qo, C, p->hq) || !make_k_map(&ta.ql_map, Ql, C, p->hq) ||
      !make_k_map(&ta.ko_map, Ko, L, p->hkv) || !make_k_map(&ta.kl_map, Kl, L, p->hkv) ||
      !make_v_map(&ta.v_map, vcache, L, p->hkv, 1))
    return BF_ERR_CUDA;
  ta.out = static_cast<bf16*>(out);
  ta.lse = lse;
  ta.L = L;
  ta.hq = p->hq;
  ta.hkv = p->hkv;
  ta.batch = 1;
  ta.w0 = kind != bf::tc2::KIND_PLAIN ? p->w0 : L;
  ta.q_off = P0;
  ta.Lq = C;
  ta.scale_log2 = scale_log2(p);
  ta.test_skip_fill = g_test_skip_fill;
  constexpr int smem = bf::attn_tc2_smem_bytes();
  const long long n_cta = static_cast<long long>((C + bf::tc::BM - 1) / bf::tc::BM) * (p->hq / 2);
  auto kern = kind == bf::tc2::KIND_BIFOCAL  ? bf::attn_tc2_kernel<bf::tc2::KIND_BIFOCAL, false>
              : kind == bf::tc2::KIND_WINDOW ? bf::attn_tc2_kernel<bf::tc2::KIND_WINDOW, false>
                                        : bf::attn_tc2_kernel<bf::tc2::KIND_PLAIN, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) {
    kern<<<static_cast<unsigned>(n_cta), bf::tc2::NTHREADS2, smem, st>>>(ta);
    e = cudaGetLastError();
  }
  return e == cudaSuccess ? BF_OK : BF_ERR_CUDA;
}

bf_status_t prefill_impl(bool bifocal_api, const void* q, const void* k, const void* v, int32_t dtype, int32_t batch,
                         int32_t L, const bf_params_t* p, void* out, float* lse, void* kcache_out, void* vcache_out,
                         void* workspace, size_t ws_bytes, void* stream) {
  // validate everything before the first launch
  bf_status_t s = check_params(p, bifocal_api);
  if (s != BF_OK) return s;
  if (!q || !k || !v || !out) return BF_ERR_INVALID;
  if (!aligned(out, 16) || (lse && !aligned(lse, 4))) return BF_ERR_INVALID;
  s = prefill_rope_impl(bifocal_api, q, k, v, dtype, batch, L, p, kcache_out, vcache_out, workspace, ws_bytes, stream);
  if (s != BF_OK) return s;
  PrefillPlan plan;
  s = plan_prefill(bifocal_api, dtype, batch, L, p, workspace, ws_bytes, &plan);
  if (s != BF_OK) return s;
  if (plan.fused)
    return fused_attention(plan.kind, q, k, false, v, batch, L, 0, L, plan.G, p, plan.rope, out, lse,
                           static_cast<cudaStream_t>(stream));
  return prefill_attention_impl(bifocal_api, v, dtype, batch, L, p, out, lse, workspace, ws_bytes, stream);
}

// ------------------------------------------------------------------ decode
struct DecodeLayout {
  size_t part_o, part_ml, total;
};

// The split-KV partial kernel; the test instantiation only while a skipped stage is armed.
template <int D, bool TEST>
cudaError_t launch_partial_t(dim3 grid, cudaStream_t st, const bf::DecodeArgs& da) {
  constexpr int smem = bf::decode_smem_bytes<D>();
  // The shared-memory limit is an attribute of the kernel in the current context: set it once
  // per device rather than on every step, and again if a launch is refused (a context made anew
  // after a device reset starts without it).
  static std::atomic<bool> set_on[64];
  auto set_attr = [&]() {
    return cudaFuncSetAttribute(bf::decode_partial_kernel<D, TEST>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  };
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const bool known = dev >= 0 && dev < 64 && set_on[dev].load(std::memory_order_relaxed);
  if (!known) {
    const cudaError_t e = set_attr();
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) set_on[dev].store(true, std::memory_order_relaxed);
  }
  cudaError_t e = launch_pdl(bf::decode_partial_kernel<D, TEST>, grid, dim3(bf::decode_threads<D>()), smem, st, da);
  if (e != cudaSuccess && known) {
    (void)cudaGetLastError();
    if (set_attr() == cudaSuccess)
      e = launch_pdl(bf::decode_partial_kernel<D, TEST>, grid, dim3(bf::decode_threads<D>()), smem, st, da);
  }
  return e;
}

cudaError_t launch_partial(int D, dim3 grid, cudaStream_t st, const bf::DecodeArgs& da) {
  const bool test = da.test_skip_stage > 0;
  if (D == 128) return test ? launch_partial_t<128, true>(grid, st, da) : launch_partial_t<128, false>(grid, st, da);
  return test ? launch_partial_t<64, true>(grid, st, da) : launch_partial_t<64, false>(grid, st, da);
}

// The combine (PDL-chained to the partial kernel), with the smallest load batch NB that covers
// a warp's share of the at most n_split partials per head in one pass.
template <int D, int NB>
cudaError_t launch_combine_t(dim3 grid, cudaStream_t st, const float* po, const float* pml, int n_split, int hq,
                             bf16* out, float* lse, const int* seq_lens, int split_len, int stride, int max_len) {
  return launch_pdl(bf::decode_combine_kernel<D, NB>, grid, dim3(32 * bf::COMBINE_WARPS), 0, st, po, pml, n_split,
                    hq, out, lse, seq_lens, split_len, stride, max_len);
}

template <int D>
cudaError_t launch_combine_d(dim3 grid, cudaStream_t st, const float* po, const float* pml, int n_split, int hq,
                             bf16* out, float* lse, const int* seq_lens, int split_len, int stride, int max_len) {
  const int per_warp = (n_split + bf::COMBINE_WARPS - 1) / bf::COMBINE_WARPS;
  if (per_warp <= 2)
    return launch_combine_t<D, 2>(grid, st, po, pml, n_split, hq, out, lse, seq_lens, split_len, stride, max_len);
  if (per_warp <= 4)
    return launch_combine_t<D, 4>(grid, st, po, pml, n_split, hq, out, lse, seq_lens, split_len, stride, max_len);
  if (per_warp <= 8)
    return launch_combine_t<D, 8>(grid, st, po, pml, n_split, hq, out, lse, seq_lens, split_len, stride, max_len);
  return launch_combine_t<D, 16>(grid, st, po, pml, n_split, hq, out, lse, seq_lens, split_len, stride, max_len);
}

cudaError_t launch_combine(int D, dim3 grid, cudaStream_t st, const float* po, const float* pml, int n_split, int hq,
                           bf16* out, float* lse, const int* seq_lens, int split_len, int stride, int max_len) {
  return D == 128 ? launch_combine_d<128>(grid, st, po, pml, n_split, hq, out, lse, seq_lens, split_len, stride, max_len)
                  : launch_combine_d<64>(grid, st, po, pml, n_split, hq, out, lse, seq_lens, split_len, stride, max_len);
}

DecodeLayout decode_layout(int L_max, const bf_params_t* p) {
  DecodeLayout w{};
  // one partial per CTA split (the two consumer warps of a kv head merge theirs in the CTA)
  const int splits = std::min(kMaxSplits, (L_max + bf::dec::KB - 1) / bf::dec::KB);
  w.part_o = 0;
  w.part_ml = align256(static_cast<size_t>(splits) * p->hq * p->head_dim * 4);
  w.total = w.part_ml + align256(static_cast<size_t>(splits) * p->hq * 2 * 4);
  return w;
}

bf_status_t decode_impl(bool bifocal_api, const void* q, const void* k_new, const void* v_new, void* kcache,
                        void* vcache, int32_t cap, int32_t L, const bf_params_t* p, void* out, float* lse,
                        void* workspace, size_t ws_bytes, void* stream) {
  bf_status_t s = check_params(p, bifocal_api);
  if (s != BF_OK) return s;
  if (!q || !k_new || !v_new || !kcache || !vcache || !out) return BF_ERR_INVALID;
  if (L < 1 || cap < L) return BF_ERR_INVALID;
  if (p->hq / p->hkv > bf::dec::MAX_G) return BF_ERR_UNSUPPORTED;
  if (!aligned(kcache, 16) || !aligned(vcache, 16) || !aligned(q, 16) || !aligned(k_new, 16) || !aligned(v_new, 16))
    return BF_ERR_INVALID;
  const bool window = bifocal_api && (p->flags & BF_FLAG_WINDOW);
  if (window && p->w0 < 1) return BF_ERR_INVALID;
  const DecodeLayout lay = decode_layout(L, p);
  if (!workspace || !aligned(workspace, 256) || ws_bytes < lay.total) return BF_ERR_WORKSPACE;

  const int D = p->head_dim;
  const int G = bifocal_api ? factor(L, p->w_pretrained) : 1;
  // BF_FLAG_FORCE_BIFOCAL runs the two-branch kernel whatever G and w0 are, as in prefill
  const bool bif = !window && bifocal_api && ((p->flags & BF_FLAG_FORCE_BIFOCAL) || (G > 1 && p->w0 < L));
  const int key0 = window ? std::max(0, L - p->w0) : 0;  // a window reads keys L - w0 .. L - 1 only
  const Rope rope = make_rope(p->rope_theta, D, G);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  // 1. append the new token
  bf::AppendArgs ap{};
  ap.k_new = static_cast<const bf16*>(k_new);
  ap.v_new = static_cast<const bf16*>(v_new);
  ap.kcache = static_cast<bf16*>(kcache);
  ap.vcache = static_cast<bf16*>(vcache);
  ap.hkv = p->hkv;
  ap.p = L - 1;
  std::memcpy(ap.omega, rope.omega, sizeof(ap.omega));
  // launched early (PDL): it waits in the kernel for whatever ran before it on the stream
  cudaError_t ea = D == 128 ? launch_pdl(bf::decode_append_kernel<128>, dim3(p->hkv), dim3(32), 0, st, ap)
                            : launch_pdl(bf::decode_append_kernel<64>, dim3(p->hkv), dim3(32), 0, st, ap);
  if (ea != cudaSuccess) return BF_ERR_CUDA;

  // 2. split-KV partials
  bf::DecodeArgs da;
  std::memset(&da, 0, sizeof(da));
  if (!make_cache_map(&da.kmap, kcache, cap, p->hkv, D, bf::dec::KB) ||
      !make_cache_map(&da.vmap, vcache, cap, p->hkv, D, bf::dec::KB))
    return BF_ERR_CUDA;
  const int head_groups = (p->hkv + bf::dec::HPC - 1) / bf::dec::HPC;
  const int sms = std::max(1, sm_count());
  const int target = std::max(1, std::min(kMaxSplits, sms / head_groups));
  const int n_keys = L - key0;
  int split_len = (n_keys + target - 1) / target;
  split_len = (split_len + bf::dec::KB - 1) / bf::dec::KB * bf::dec::KB;
  const int n_split = (n_keys + split_len - 1) / split_len;
  da.q = static_cast<const bf16*>(q);
  da.part_o = reinterpret_cast<float*>(ws + lay.part_o);
  da.part_ml = reinterpret_cast<float*>(ws + lay.part_ml);
  da.L = L;
  da.hq = p->hq;
  da.hkv = p->hkv;
  da.w0 = p->w0;
  da.G = G;
  da.mode = bifocal_api ? p->mode : 0;
  da.bifocal = bif ? 1 : 0;
  da.key0 = key0;
  da.split_len = split_len;
  da.n_split = n_split;
  da.scale_log2 = scale_log2(p);
  da.test_skip_stage = g_test_skip_stage;
  std::memcpy(da.omega, rope.omega, sizeof(da.omega));
  std::memcpy(da.omega_long, rope.omega_long, sizeof(da.omega_long));
  std::memcpy(da.omega_corr, rope.omega_corr, sizeof(da.omega_corr));
  const dim3 grid(n_split, head_groups);
  cudaError_t e;
  // the partial and combine kernels overlap their launch with the kernel before them
  e = launch_partial(D, grid, st, da);
  if (e != cudaSuccess) return BF_ERR_CUDA;

  // 3. combine
  e = launch_combine(D, dim3(p->hq, D / 32), st, da.part_o, da.part_ml, n_split, p->hq, static_cast<bf16*>(out), lse,
                     nullptr, 0, 0, 0);
  return e == cudaSuccess ? BF_OK : BF_ERR_CUDA;
}

// ------------------------------------------------------------------ allocation-free decode
// Static scratch for bifocal_decode_noalloc: holds the split-KV partials. Every call shares
// it; overlapping calls race (documented in the header).
__device__ __align__(256) uint8_t g_noalloc_scratch[BIFOCAL_NOALLOC_SCRATCH_BYTES];

// Host code cannot use the array's name as a device address: look the address up once per
// device, with that device current. The address belongs to the device's current context; a
// device reset (or a primary context released and created again) gives the module a new
// address, so the cached one is kept together with the unique id of the context it was read
// in, and looked up again when the current context is another one.
constexpr int kMaxDevices = 64;
struct NoallocEntry {
  void* ptr;
  unsigned long long ctx_id;
};
NoallocEntry g_noalloc[kMaxDevices] = {};
std::mutex g_noalloc_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the current context (0 when it cannot be read: then the address is looked up
// on every call, which costs a driver call but is always right).
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
        qa == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
        qb == cudaDriverEntryPointSuccess) {
      get_cur = reinterpret_cast<CtxGetCurrentFn>(a);
      get_id = reinterpret_cast<CtxGetIdFn>(b);
    }
  });
  if (!get_cur || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

void* noalloc_scratch_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoallocEntry& e = g_noalloc[dev];
  if (cudaFree(nullptr) != cudaSuccess) return nullptr;  // makes the device's primary context current
  const unsigned long long id = current_ctx_id();
  if (!e.ptr || id == 0 || e.ctx_id != id) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
    e.ptr = ptr;
    e.ctx_id = id;
  }
  return e.ptr;
}

}  // namespace

// ------------------------------------------------------------------ batched decode over a paged cache
// Partial rows per sequence: one per split, splits <= min(kMaxSplits, ceil(max_len / KB)).
int paged_parts_stride(int max_len) { return std::min(kMaxSplits, (max_len + bf::dec::KB - 1) / bf::dec::KB); }

size_t paged_workspace(int batch, int max_len, const bf_params_t* p) {
  const size_t rows = static_cast<size_t>(batch) * paged_parts_stride(max_len) * p->hq;
  return align256(rows * p->head_dim * 4) + align256(rows * 2 * 4);
}

bf_status_t decode_paged_impl(const void* q, const void* k_new, const void* v_new, void* kpool, void* vpool,
                              int32_t pool_pages, int32_t page_size, const int32_t* block_table, int32_t max_pages,
                              const int32_t* seq_lens, int32_t max_len, int32_t batch, const bf_params_t* p,
                              void* out, float* lse, void* workspace, size_t ws_bytes, void* stream) {
  bf_status_t s = check_params(p, true);
  if (s != BF_OK) return s;
  if (!q || !k_new || !v_new || !kpool || !vpool || !block_table || !seq_lens || !out) return BF_ERR_INVALID;
  if (batch < 1 || pool_pages < 1 || max_pages < 1 || max_len < 1) return BF_ERR_INVALID;
  if (page_size < bf::dec::KB || page_size % bf::dec::KB) return BF_ERR_INVALID;
  if (static_cast<int64_t>(max_pages) * page_size < max_len ||
      static_cast<int64_t>(pool_pages) * page_size > 0x7fffffffLL)
    return BF_ERR_INVALID;
  if (p->hq / p->hkv > bf::dec::MAX_G) return BF_ERR_UNSUPPORTED;
  if (p->flags & BF_FLAG_WINDOW) return BF_ERR_UNSUPPORTED;
  if (!aligned(kpool, 16) || !aligned(vpool, 16) || !aligned(q, 16) || !aligned(k_new, 16) || !aligned(v_new, 16) ||
      !aligned(block_table, 4) || !aligned(seq_lens, 4) || !aligned(out, 16) || (lse && !aligned(lse, 4)))
    return BF_ERR_INVALID;
  if (!workspace || !aligned(workspace, 256) || ws_bytes < paged_workspace(batch, max_len, p)) return BF_ERR_WORKSPACE;

  const int D = p->head_dim;
  const Rope rope = make_rope(p->rope_theta, D, 1);  // omega only: G is each sequence's own
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int stride = paged_parts_stride(max_len);
  const size_t rows = static_cast<size_t>(batch) * stride * p->hq;
  float* part_o = reinterpret_cast<float*>(ws);
  float* part_ml = reinterpret_cast<float*>(ws + align256(rows * D * 4));

  // 1. append every sequence's new token at its own position
  bf::AppendArgs ap{};
  ap.k_new = static_cast<const bf16*>(k_new);
  ap.v_new = static_cast<const bf16*>(v_new);
  ap.kcache = static_cast<bf16*>(kpool);
  ap.vcache = static_cast<bf16*>(vpool);
  ap.hkv = p->hkv;
  ap.seq_lens = seq_lens;
  ap.block_table = block_table;
  ap.max_pages = max_pages;
  ap.page_size = page_size;
  ap.pool_pages = pool_pages;
  ap.max_len = max_len;
  std::memcpy(ap.omega, rope.omega, sizeof(ap.omega));
  cudaError_t ea = D == 128 ? launch_pdl(bf::decode_append_kernel<128>, dim3(p->hkv, batch), dim3(32), 0, st, ap)
                            : launch_pdl(bf::decode_append_kernel<64>, dim3(p->hkv, batch), dim3(32), 0, st, ap);
  if (ea != cudaSuccess) return BF_ERR_CUDA;

  // 2. split-KV partials: one split length for the batch (from max_len), a grid of about one
  //    CTA per SM in total; CTAs past a shorter sequence's end leave at once
  bf::DecodeArgs da;
  std::memset(&da, 0, sizeof(da));
  const int cap = pool_pages * page_size;
  if (!make_cache_map(&da.kmap, kpool, cap, p->hkv, D, bf::dec::KB) ||
      !make_cache_map(&da.vmap, vpool, cap, p->hkv, D, bf::dec::KB))
    return BF_ERR_CUDA;
  const int head_groups = (p->hkv + bf::dec::HPC - 1) / bf::dec::HPC;
  const int sms = std::max(1, sm_count());
  const int target = std::max(1, std::min(kMaxSplits, sms / (head_groups * batch)));
  int split_len = (max_len + target - 1) / target;
  split_len = (split_len + bf::dec::KB - 1) / bf::dec::KB * bf::dec::KB;
  const int n_split = (max_len + split_len - 1) / split_len;
  da.q = static_cast<const bf16*>(q);
  da.part_o = part_o;
  da.part_ml = part_ml;
  da.L = max_len;
  da.hq = p->hq;
  da.hkv = p->hkv;
  da.w0 = p->w0;
  da.mode = p->mode;
  da.split_len = split_len;
  da.n_split = n_split;
  da.scale_log2 = scale_log2(p);
  std::memcpy(da.omega, rope.omega, sizeof(da.omega));
  da.seq_lens = seq_lens;
  da.block_table = block_table;
  da.max_pages = max_pages;
  da.page_size = page_size;
  da.w_pretrained = p->w_pretrained;
  da.force_bifocal = (p->flags & BF_FLAG_FORCE_BIFOCAL) ? 1 : 0;
  da.parts_stride = stride;
  da.pool_pages = pool_pages;
  da.test_skip_stage = g_test_skip_stage;
  const dim3 grid(n_split, head_groups, batch);
  cudaError_t e;
  e = launch_partial(D, grid, st, da);
  if (e != cudaSuccess) return BF_ERR_CUDA;

  // 3. combine per sequence
  e = launch_combine(D, dim3(p->hq, D / 32, batch), st, part_o, part_ml, n_split, p->hq, static_cast<bf16*>(out), lse,
                     seq_lens, split_len, stride, max_len);
  return e == cudaSuccess ? BF_OK : BF_ERR_CUDA;
}

// ------------------------------------------------------------------ batched chunks over a paged cache
bf_status_t chunk_paged_impl(const void* q, const void* k, const void* v, int32_t batch, const int32_t* chunk_lens,
                             const int32_t* cached_lens, const bf_params_t* p, void* kpool, void* vpool,
                             int32_t pool_pages, int32_t page_size, const int32_t* block_table, int32_t max_pages,
                             void* out, float* lse, void* stream) {
  bf_status_t s = check_params(p, true);
  if (s != BF_OK) return s;
  if (!q || !k || !v || !kpool || !vpool || !block_table || !out || !chunk_lens || !cached_lens) return BF_ERR_INVALID;
  if (batch < 1 || pool_pages < 1 || max_pages < 1) return BF_ERR_INVALID;
  if (batch > bf::tc2::kMaxSeqs) return BF_ERR_UNSUPPORTED;
  if (page_size < 16 || page_size % 16 || (128 % page_size && page_size % 128)) return BF_ERR_INVALID;
  if (static_cast<int64_t>(pool_pages) * page_size > 0x7fffffffLL) return BF_ERR_INVALID;
  const int D = p->head_dim, g = p->hq / p->hkv;
  if (D != 128 || p->hq % 2 || g % 2 || (p->flags & BF_FLAG_MMA_SYNC)) return BF_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(kpool, 16) || !aligned(vpool, 16) ||
      !aligned(out, 16) || !aligned(block_table, 4) || (lse && !aligned(lse, 4)))
    return BF_ERR_INVALID;
  const bool window = (p->flags & BF_FLAG_WINDOW) != 0;
  if (window && p->w0 < 1) return BF_ERR_INVALID;
  int64_t total = 0;
  int order[bf::tc2::kMaxSeqs];
  double work[bf::tc2::kMaxSeqs];
  for (int i = 0; i < batch; ++i) {
    const int64_t P0 = cached_lens[i], C = chunk_lens[i];
    if (P0 < 0 || C < 1 || P0 + C > static_cast<int64_t>(max_pages) * page_size) return BF_ERR_INVALID;
    total += C;
    order[i] = i;
    work[i] = static_cast<double>(C) * (static_cast<double>(P0) + 0.5 * C);  // causal pairs of the chunk
  }
  if (total > 0x7fffffffLL) return BF_ERR_INVALID;
  // launch order: the most work first, so the tail of the grid is light
  std::sort(order, order + batch, [&](int x, int y) { return work[x] > work[y]; });
  const int T = static_cast<int>(total);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Rope rope = make_rope(p->rope_theta, D, 1);

  // 1. every chunk's keys (original RoPE, bf16) and values into its pages
  bf::PrepassArgs pa{};
  pa.q = q;
  pa.k = k;
  pa.v = v;
  pa.batch = 1;
  pa.L = T;
  pa.Lk = T;
  pa.Lc = 0;
  pa.hq = p->hq;
  pa.hkv = p->hkv;
  pa.G = 1;
  pa.keys_only = 1;
  pa.kcache = static_cast<bf16*>(kpool);
  pa.vcache = static_cast<bf16*>(vpool);
  pa.nseq = batch;
  pa.block_table = block_table;
  pa.max_pages = max_pages;
  pa.page_size = page_size;
  pa.pool_pages = pool_pages;
  int row = 0;
  for (int i = 0; i < batch; ++i) {
    pa.seq_id[i] = i;
    pa.seq_P0[i] = cached_lens[i];
    pa.seq_C[i] = chunk_lens[i];
    pa.seq_qrow[i] = row;
    row += chunk_lens[i];
  }
  std::memcpy(pa.omega, rope.omega, sizeof(pa.omega));
  bf::rope_prepass_kernel<bf16, 128><<<static_cast<unsigned>((T + 7) / 8), 256, 0, st>>>(pa);
  if (cudaGetLastError() != cudaSuccess) return BF_ERR_CUDA;

  // 2. the fused attention over every sequence's chunk, keys re-phased in the tile loads
  bf::Tc2Args ta;
  std::memset(&ta, 0, sizeof(ta));
  const int seg = std::min(page_size, 128);
  const int pool_rows = pool_pages * page_size;
  if (!make_v_map(&ta.qo_map, q, T, p->hq, 1) || !make_v_map(&ta.ko_map, kpool, pool_rows, p->hkv, 1, seg) ||
      !make_v_map(&ta.v_map, vpool, pool_rows, p->hkv, 1, seg))
    return BF_ERR_CUDA;
  ta.out = static_cast<bf16*>(out);
  ta.lse = lse;
  ta.hq = p->hq;
  ta.hkv = p->hkv;
  ta.batch = 1;
  ta.w0 = p->w0;
  ta.scale_log2 = scale_log2(p);
  ta.src.cache = 1;
  ta.src.mode = p->mode;
  ta.src.G = 1;
  std::memcpy(ta.src.omega, rope.omega, sizeof(ta.src.omega));
  ta.test_skip_fill = g_test_skip_fill;
  ta.nseq = batch;
  ta.total_rows = T;
  ta.block_table = block_table;
  ta.max_pages = max_pages;
  ta.page_size = page_size;
  ta.seg_rows = seg;
  ta.pool_pages = pool_pages;
  int tiles = 0;
  for (int si = 0; si < batch; ++si) {
    const int i = order[si];
    ta.tile_start[si] = tiles;
    ta.seq_id[si] = i;
    ta.seq_P0[si] = cached_lens[i];
    ta.seq_C[si] = chunk_lens[i];
    ta.seq_G[si] = factor(static_cast<int64_t>(cached_lens[i]) + chunk_lens[i], p->w_pretrained);
    ta.seq_qrow[si] = pa.seq_qrow[i];
    tiles += (chunk_lens[i] + bf::tc::BM - 1) / bf::tc::BM;
  }
  ta.tile_start[batch] = tiles;
  const long long n_cta = static_cast<long long>(tiles) * (p->hq / 2);
  // one kernel kind for the batch: a sequence with G = 1 or w0 >= its length takes the two-branch
  // kernel as with BF_FLAG_FORCE_BIFOCAL (its long-range forms equal the original ones, or it has
  // no long-range visit)
  const int kind = window ? bf::tc2::KIND_WINDOW : bf::tc2::KIND_BIFOCAL;
  return launch_tc2(kind, true, ta, n_cta, st) == cudaSuccess ? BF_OK : BF_ERR_CUDA;
}

extern "C" {

bf_status_t bifocal_prefill_chunk_paged(const void* q, const void* k, const void* v, int32_t batch,
                                        const int32_t* chunk_lens, const int32_t* cached_lens, const bf_params_t* p,
                                        void* kpool, void* vpool, int32_t pool_pages, int32_t page_size,
                                        const int32_t* block_table, int32_t max_pages, void* out, float* lse,
                                        void* stream) {
  return chunk_paged_impl(q, k, v, batch, chunk_lens, cached_lens, p, kpool, vpool, pool_pages, page_size,
                          block_table, max_pages, out, lse, stream);
}

int32_t bifocal_factor(int64_t L, int32_t w_pretrained) {
  if (L < 0 || w_pretrained < 1) return -1;
  return factor(L, w_pretrained);
}

size_t bifocal_prefill_workspace_size(int32_t dtype, int32_t batch, int32_t L, const bf_params_t* p) {
  if (check_params(p, false) != BF_OK || batch < 1 || L < 1) return 0;
  if (dtype != BF_DTYPE_BF16 && dtype != BF_DTYPE_FP32) return 0;
  return prefill_layout(dtype, batch, L, p).total;
}

bf_status_t bifocal_prefill(const void* q, const void* k, const void* v, int32_t dtype, int32_t batch, int32_t L,
                            const bf_params_t* p, void* out, float* lse, void* kcache_out, void* vcache_out,
                            void* workspace, size_t ws_bytes, void* stream) {
  return prefill_impl(true, q, k, v, dtype, batch, L, p, out, lse, kcache_out, vcache_out, workspace, ws_bytes,
                      stream);
}

size_t bifocal_decode_paged_workspace_size(int32_t batch, int32_t max_len, const bf_params_t* p) {
  if (check_params(p, true) != BF_OK || batch < 1 || max_len < 1) return 0;
  return paged_workspace(batch, max_len, p);
}

bf_status_t bifocal_decode_paged(const void* q, const void* k_new, const void* v_new, void* kpool, void* vpool,
                                 int32_t pool_pages, int32_t page_size, const int32_t* block_table, int32_t max_pages,
                                 const int32_t* seq_lens, int32_t max_len, int32_t batch, const bf_params_t* p,
                                 void* out, float* lse, void* workspace, size_t ws_bytes, void* stream) {
  return decode_paged_impl(q, k_new, v_new, kpool, vpool, pool_pages, page_size, block_table, max_pages, seq_lens,
                           max_len, batch, p, out, lse, workspace, ws_bytes, stream);
}

size_t bifocal_prefill_chunk_workspace_size(int32_t P0, int32_t C, const bf_params_t* p) {
  if (check_params(p, true) != BF_OK || P0 < 0 || C < 1 || static_cast<int64_t>(P0) + C > 0x7fffffff) return 0;
  return chunk_layout(P0, C, p, BF_DTYPE_BF16).total;
}

bf_status_t bifocal_prefill_chunk(const void* q, const void* k, const void* v, int32_t dtype, int32_t P0, int32_t C,
                                  const bf_params_t* p, void* kcache, void* vcache, int32_t cap, void* out, float* lse,
                                  void* workspace, size_t ws_bytes, void* stream) {
  return chunk_impl(q, k, v, dtype, P0, C, p, kcache, vcache, cap, out, lse, workspace, ws_bytes, stream);
}

bf_status_t bifocal_prefill_rope(const void* q, const void* k, const void* v, int32_t dtype, int32_t batch,
                                 int32_t L, const bf_params_t* p, void* kcache_out, void* vcache_out, void* workspace,
                                 size_t ws_bytes, void* stream) {
  return prefill_rope_impl(true, q, k, v, dtype, batch, L, p, kcache_out, vcache_out, workspace, ws_bytes, stream);
}

bf_status_t bifocal_prefill_rope_qknorm(const void* q, const void* k, const void* v, int32_t dtype, int32_t batch,
                                        int32_t L, const bf_params_t* p, const void* q_norm_w, const void* k_norm_w,
                                        float eps, void* kcache_out, void* vcache_out, void* workspace,
                                        size_t ws_bytes, void* stream) {
  if (!q_norm_w || !k_norm_w || !(eps >= 0.f) || !std::isfinite(eps)) return BF_ERR_INVALID;
  const size_t align_in = dtype == BF_DTYPE_FP32 ? 32 : 16;
  if (!aligned(q_norm_w, align_in) || !aligned(k_norm_w, align_in)) return BF_ERR_INVALID;
  return prefill_rope_impl(true, q, k, v, dtype, batch, L, p, kcache_out, vcache_out, workspace, ws_bytes, stream,
                           q_norm_w, k_norm_w, eps);
}

bf_status_t bifocal_prefill_attention(const void* v, int32_t dtype, int32_t batch, int32_t L, const bf_params_t* p,
                                      void* out, float* lse, void* workspace, size_t ws_bytes, void* stream) {
  return prefill_attention_impl(true, v, dtype, batch, L, p, out, lse, workspace, ws_bytes, stream);
}

bf_status_t rope_causal_prefill(const void* q, const void* k, const void* v, int32_t dtype, int32_t batch, int32_t L,
                                const bf_params_t* p, void* out, float* lse, void* kcache_out, void* vcache_out,
                                void* workspace, size_t ws_bytes, void* stream) {
  return prefill_impl(false, q, k, v, dtype, batch, L, p, out, lse, kcache_out, vcache_out, workspace, ws_bytes,
                      stream);
}

size_t bifocal_decode_workspace_size(int32_t L_max, const bf_params_t* p) {
  if (check_params(p, false) != BF_OK || L_max < 1) return 0;
  return decode_layout(L_max, p).total;
}

bf_status_t bifocal_decode(const void* q, const void* k_new, const void* v_new, void* kcache, void* vcache,
                           int32_t cap, int32_t L, const bf_params_t* p, void* out, float* lse, void* workspace,
                           size_t ws_bytes, void* stream) {
  return decode_impl(true, q, k_new, v_new, kcache, vcache, cap, L, p, out, lse, workspace, ws_bytes, stream);
}

bf_status_t bifocal_decode_noalloc(const void* q, const void* k_new, const void* v_new, void* kcache, void* vcache,
                                   int32_t cap, int32_t L, const bf_params_t* p, void* out, float* lse, void* stream) {
  bf_status_t s = check_params(p, true);
  if (s != BF_OK) return s;
  if (L < 1 || cap < L) return BF_ERR_INVALID;
  const size_t need = decode_layout(L, p).total;
  if (need > BIFOCAL_NOALLOC_SCRATCH_BYTES) return BF_ERR_WORKSPACE;
  void* scratch = noalloc_scratch_ptr();
  if (!scratch) return BF_ERR_CUDA;
  return decode_impl(true, q, k_new, v_new, kcache, vcache, cap, L, p, out, lse, scratch,
                     BIFOCAL_NOALLOC_SCRATCH_BYTES, stream);
}

bf_status_t rope_causal_decode(const void* q, const void* k_new, const void* v_new, void* kcache, void* vcache,
                               int32_t cap, int32_t L, const bf_params_t* p, void* out, float* lse,
                               void* workspace, size_t ws_bytes, void* stream) {
  return decode_impl(false, q, k_new, v_new, kcache, vcache, cap, L, p, out, lse, workspace, ws_bytes, stream);
}

const char* bifocal_status_string(int32_t status) {
  switch (status) {
    case BF_OK: return "ok";
    case BF_ERR_INVALID: return "invalid argument";
    case BF_ERR_UNSUPPORTED: return "unsupported configuration";
    case BF_ERR_CUDA: return "CUDA error";
    case BF_ERR_TIMEOUT: return "device-side wait timed out";
    case BF_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case BF_ERR_NO_DEVICE: return "no suitable CUDA device";
    case BF_ERR_RANGE: return "an fp16 QK^T operand was not finite after rounding (|x| >= 65520, inf or NaN)";
    case BF_ERR_INDEX: return "a sequence length or block-table entry in device memory was out of range";
    default: return "unknown status";
  }
}

bf_status_t bifocal_last_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return BF_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, bf::g_device_status, sizeof(int)) != cudaSuccess) return BF_ERR_CUDA;
  if (v == 0) return BF_OK;
  const int zero = 0;
  if (cudaMemcpyToSymbol(bf::g_device_status, &zero, sizeof(int)) != cudaSuccess) return BF_ERR_CUDA;
  switch (v & 0xff) {
    case bf::kDevRange: return BF_ERR_RANGE;
    case bf::kDevIndex: return BF_ERR_INDEX;
    default: return BF_ERR_TIMEOUT;
  }
}

bf_status_t bifocal_test_set_fault(int32_t kind, int32_t arg, int64_t wait_limit_ns) {
  if (kind < BF_FAULT_NONE || kind > BF_FAULT_DECODE_SKIP_STAGE || wait_limit_ns < 0) return BF_ERR_INVALID;
  if (kind != BF_FAULT_NONE && arg < 0) return BF_ERR_INVALID;
  if (cudaDeviceSynchronize() != cudaSuccess) return BF_ERR_CUDA;  // no launch in flight sees a half-set control
  const unsigned long long lim = wait_limit_ns > 0 ? static_cast<unsigned long long>(wait_limit_ns) : 2000000000ull;
  if (cudaMemcpyToSymbol(bf::g_wait_limit_ns, &lim, sizeof(lim)) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess)
    return BF_ERR_CUDA;
  g_test_skip_fill = kind == BF_FAULT_PREFILL_SKIP_FILL ? arg + 1 : 0;
  g_test_skip_stage = kind == BF_FAULT_DECODE_SKIP_STAGE ? arg + 1 : 0;
  return BF_OK;
}

int32_t bifocal_device_status_word(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, bf::g_device_status, sizeof(int)) != cudaSuccess) return -1;
  return v;
}

const char* bifocal_build_info(void) {
  return "bifocal sm_100a: rope pass; prefill D=128 tcgen05/TMEM/TMA (D=64 and BF_FLAG_MMA_SYNC: mma.sync); "
         "decode split-KV (TMA + mma.sync)";
}

}  // extern "C"
