// RoPE pre-pass of the prefill: one HBM pass over the raw q and k.
//
// For every position p it evaluates the rotation angles once (fp64 product and range
// reduction, see angle_cos_sin) and applies them to every head:
//   Qo = R_orig(p) q,  Ql = R_long(p) q   -> [b, hq,  L, D] fp16 (head-major tiles)
//   Ko = R_orig(p) k,  Kl = R_long(p) k   -> [b, hkv, L, D] fp16
// The rotated forms are the QK^T operands. They are rounded once, to fp16 rather than
// bf16: same tensor-core rate, 8x smaller rounding error, so a score is off by ~2e-4
// instead of ~3e-3 (which would exceed a 1e-3 LSE bound on rows that see few keys).
// R_orig rotates pair k by p * omega_k; R_long by p * omega_k / G (frequency
// interpolation) or floor(p / G) * omega_k (position aliasing) - the two long-range
// forms named by the ablation of the ai-feeds summary of Jet-Long (实验, key findings).
// Ko is also the decode cache (keys under the original RoPE) and is written to the
// caller's kcache in [b, Lc, hkv, D] when asked. fp32 inputs are rounded to bf16 here.
// A chunk over an existing cache passes its first absolute position in pos0: the angles,
// the key rows and the cache rows are those of positions pos0 .. pos0 + L - 1.
// With q_norm_w / k_norm_w the pass first applies the per-head RMS norm of the model's
// attention block (Qwen3 normalises every query and key head over D with a learned weight
// before RoPE), so the step before the path costs no extra pass over q and k.
//
// cache_rephase_kernel prepares the cached part of a chunked prefill: the cache holds
// keys under the original RoPE (bf16), so Ko is their fp16 copy (exact: a bf16 value
// of normal magnitude has 8 significant bits, fp16 11), and Kl re-phases them by the
// correction rotation R_long(j) R_orig(j)^-1 - angle j * omega_k * (1/G - 1) under
// frequency interpolation, (floor(j/G) - j) * omega_k under position aliasing (the
// rotation applied to cached keys in the ai-feeds summary of Jet-Long, 方法 key module 3).
#pragma once
#include "common.cuh"

namespace bf {

struct PrepassArgs {
  const void* q;
  const void* k;
  const void* v;
  int batch, L, hq, hkv;  // L rows of q, k, v per batch (a full prompt, or a chunk)
  int pos0;               // absolute position of row 0 (0, or the cached length for a chunk)
  int Lk;                 // rows of Ko / Kl per (batch, kv head): pos0 + L for a chunk
  int Lc;                 // rows of kcache / vcache per batch
  int G;
  int mode;       // 0 = frequency interpolation, 1 = position aliasing
  int need_long;  // write Ql / Kl
  int keys_only;  // skip q: only the cache rows (kcache / vcache) and the key forms that are non-null
  __half* Qo;
  __half* Ql;
  __half* Ko;
  __half* Kl;
  __nv_bfloat16* Vb;       // bf16 copy of v in [b, L, hkv, D] (fp32 inputs only), else null
  __nv_bfloat16* kcache;   // optional [b, L, hkv, D]
  __nv_bfloat16* vcache;   // optional [b, L, hkv, D]
  double omega[64];        // omega_k = theta^(-2k/D)
  double omega_long[64];   // omega_k / G (frequency interpolation)
  // optional per-head RMS norm before the rotation (Qwen3's q_norm / k_norm): x <- x *
  // rsqrt(mean_d(x^2) + eps) * w[d], weights [D] in the input dtype; null = no norm
  const void* q_norm_w;
  const void* k_norm_w;
  float norm_eps;
  // A batch of chunks appended to a paged cache (keys_only, nseq > 0; batch 1, L = the packed
  // rows): packed row g belongs to entry s with seq_qrow[s] <= g < seq_qrow[s] + seq_C[s], at
  // position seq_P0[s] + g - seq_qrow[s] of the sequence whose block-table row is seq_id[s];
  // position p of it is cache row block_table[seq_id[s] * max_pages + p / page_size] *
  // page_size + p % page_size.
  int nseq;
  const int* block_table;
  int max_pages, page_size, pool_pages;  // an entry outside [0, pool_pages) is reported, its row skipped
  int seq_id[64], seq_P0[64], seq_C[64], seq_qrow[64];
};

template <typename T>
struct Vec8;  // 8 consecutive elements of T
template <>
struct Vec8<__nv_bfloat16> {
  uint4 u;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { u = *reinterpret_cast<const uint4*>(p); }
  __device__ __forceinline__ float get(int i) const {
    const uint32_t w = (&u.x)[i >> 1];
    float2 f = unpack_bf16x2(w);
    return (i & 1) ? f.y : f.x;
  }
};
template <>
struct Vec8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = reinterpret_cast<const float4*>(p)[0];
    b = reinterpret_cast<const float4*>(p)[1];
  }
  __device__ __forceinline__ float get(int i) const {
    const float* f = (i < 4) ? &a.x : &b.x;
    return f[i & 3];
  }
};

__device__ __forceinline__ void store8_f16(__half* dst, const float (&x)[8]) {
  uint4 u;
  u.x = pack_f16x2(x[0], x[1]);
  u.y = pack_f16x2(x[2], x[3]);
  u.z = pack_f16x2(x[4], x[5]);
  u.w = pack_f16x2(x[6], x[7]);
  *reinterpret_cast<uint4*>(dst) = u;
}

__device__ __forceinline__ void store8_bf16(__nv_bfloat16* dst, const float (&x)[8]) {
  uint4 u;
  u.x = pack_bf16x2(x[0], x[1]);
  u.y = pack_bf16x2(x[2], x[3]);
  u.z = pack_bf16x2(x[4], x[5]);
  u.w = pack_bf16x2(x[6], x[7]);
  *reinterpret_cast<uint4*>(dst) = u;
}

// One warp per (batch, position). Lanes form 4 groups of 8; group g handles rows
// (heads) g, g+4, ...; lane l8 of a group owns the 8 pairs [8*l8 .. 8*l8+8) for D=128
// (elements d and d + D/2), or 4 pairs for D=64 (then lanes 4..7 of a group idle on d).
template <typename Tin, int D>
__global__ void __launch_bounds__(256) rope_prepass_kernel(const __grid_constant__ PrepassArgs a) {
  constexpr int P = D / 2;
  constexpr int NPAIR = 8;               // pairs per lane slot
  constexpr int LANES_PER_ROW = P / NPAIR;  // 8 (D=128) or 4 (D=64)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long gpos = static_cast<long long>(blockIdx.x) * 8 + warp;
  if (gpos >= static_cast<long long>(a.batch) * a.L) return;
  const int b = static_cast<int>(gpos / a.L);
  const int r_in = static_cast<int>(gpos % a.L);  // row of the input
  int p = a.pos0 + r_in;                           // absolute position
  long long crow = static_cast<long long>(b) * a.Lc + p;  // row of kcache / vcache
  if (a.nseq > 0) {
    int sq = 0;
    while (sq + 1 < a.nseq && a.seq_qrow[sq + 1] <= r_in) ++sq;
    p = a.seq_P0[sq] + (r_in - a.seq_qrow[sq]);
    const int pg = a.block_table[static_cast<long long>(a.seq_id[sq]) * a.max_pages + p / a.page_size];
    if (pg < 0 || pg >= a.pool_pages) {  // the table lies: write nothing for this row
      if (lane == 0) report_status(kDevIndex, 54);
      return;
    }
    crow = static_cast<long long>(pg) * a.page_size + p % a.page_size;
  }
  const int grp = lane >> 3, l8 = lane & 7;
  if (l8 >= LANES_PER_ROW) return;
  const int k0 = l8 * NPAIR;  // first pair index this lane owns

  float co[NPAIR], so[NPAIR], cl[NPAIR], sl[NPAIR];
  const double pl = (a.mode == 0) ? static_cast<double>(p) : static_cast<double>(p / a.G);
#pragma unroll
  for (int i = 0; i < NPAIR; ++i) {
    angle_cos_sin(static_cast<double>(p) * a.omega[k0 + i], co[i], so[i]);
    if (a.need_long) {
      if (a.mode == 0)
        angle_cos_sin(pl * a.omega_long[k0 + i], cl[i], sl[i]);
      else
        angle_cos_sin(pl * a.omega[k0 + i], cl[i], sl[i]);
    } else {
      cl[i] = co[i];
      sl[i] = so[i];
    }
  }

  const Tin* qb = static_cast<const Tin*>(a.q);
  const Tin* kb = static_cast<const Tin*>(a.k);
  const Tin* vb = static_cast<const Tin*>(a.v);
  const int rows = a.hq + a.hkv;
  for (int r = (a.keys_only ? a.hq : 0) + grp; r < rows; r += 4) {
    const bool is_q = r < a.hq;
    const int h = is_q ? r : r - a.hq;
    const int H = is_q ? a.hq : a.hkv;
    const Tin* src = (is_q ? qb : kb) + ((static_cast<long long>(b) * a.L + r_in) * H + h) * D;
    Vec8<Tin> x1, x2;
    x1.load(src + k0);
    x2.load(src + P + k0);
    float xu[8], xw[8];
#pragma unroll
    for (int i = 0; i < NPAIR; ++i) {
      xu[i] = x1.get(i);
      xw[i] = x2.get(i);
    }
    const void* nw = is_q ? a.q_norm_w : a.k_norm_w;
    if (nw) {
      // RMS over the row's D elements: this lane holds 16 (D = 128) or 8 of the row's pairs'
      // elements; the row's lanes are the LANES_PER_ROW lanes of this group
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < NPAIR; ++i) ss += xu[i] * xu[i] + xw[i] * xw[i];
      const unsigned gmask = ((1u << LANES_PER_ROW) - 1u) << (grp * 8);
#pragma unroll
      for (int off = LANES_PER_ROW / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(gmask, ss, off);
      const float inv = rsqrtf(ss / D + a.norm_eps);
      Vec8<Tin> w1, w2;
      w1.load(static_cast<const Tin*>(nw) + k0);
      w2.load(static_cast<const Tin*>(nw) + P + k0);
#pragma unroll
      for (int i = 0; i < NPAIR; ++i) {
        xu[i] *= inv * w1.get(i);
        xw[i] *= inv * w2.get(i);
      }
    }
    float yo1[8], yo2[8], yl1[8], yl2[8];
#pragma unroll
    for (int i = 0; i < NPAIR; ++i) {
      const float u = xu[i], w = xw[i];
      yo1[i] = u * co[i] - w * so[i];
      yo2[i] = w * co[i] + u * so[i];
      yl1[i] = u * cl[i] - w * sl[i];
      yl2[i] = w * cl[i] + u * sl[i];
    }
    // fp16 range guard on the QK^T operands (a larger magnitude would round to inf)
    bool fin = true;
#pragma unroll
    for (int i = 0; i < NPAIR; ++i) {
      fin &= f16_ok(yo1[i]) & f16_ok(yo2[i]);
      if (a.need_long) fin &= f16_ok(yl1[i]) & f16_ok(yl2[i]);
    }
    if (!fin) report_status(kDevRange, 40);
    // head-major rows: Q has the input's L rows, K the Lk rows of keys 0 .. Lk-1
    const long long hm = is_q ? ((static_cast<long long>(b) * H + h) * a.L + r_in) * D
                              : ((static_cast<long long>(b) * H + h) * a.Lk + p) * D;
    if (__half* dst_o = is_q ? a.Qo : a.Ko) {
      store8_f16(dst_o + hm + k0, yo1);
      store8_f16(dst_o + hm + P + k0, yo2);
    }
    if (a.need_long) {
      __half* dst_l = (is_q ? a.Ql : a.Kl) + hm;
      store8_f16(dst_l + k0, yl1);
      store8_f16(dst_l + P + k0, yl2);
    }
    if (!is_q && a.kcache) {
      __nv_bfloat16* dc = a.kcache + (crow * a.hkv + h) * D;
      store8_bf16(dc + k0, yo1);
      store8_bf16(dc + P + k0, yo2);
    }
  }
  // v: bf16 copy for fp32 inputs and / or the caller's vcache
  if (a.Vb || a.vcache) {
    for (int h = grp; h < a.hkv; h += 4) {
      const long long off = ((static_cast<long long>(b) * a.L + r_in) * a.hkv + h) * D;
      const long long coff = (crow * a.hkv + h) * D;
      Vec8<Tin> x1, x2;
      x1.load(vb + off + k0);
      x2.load(vb + off + P + k0);
      float y1[8], y2[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        y1[i] = x1.get(i);
        y2[i] = x2.get(i);
      }
      if (a.Vb) {
        store8_bf16(a.Vb + off + k0, y1);
        store8_bf16(a.Vb + off + P + k0, y2);
      }
      if (a.vcache) {
        store8_bf16(a.vcache + coff + k0, y1);
        store8_bf16(a.vcache + coff + P + k0, y2);
      }
    }
  }
}

struct RephaseArgs {
  const __nv_bfloat16* kcache;  // [Lc, hkv, D], rows 0 .. P0-1 read
  int P0, hkv, Lk;              // cached rows; kv heads; rows of Ko / Kl per kv head
  int j_begin;                  // first cached row needed (0, or the window's first tile)
  int G, mode, need_long;
  __half* Ko;                   // [hkv, Lk, D]
  __half* Kl;
  double omega[64];
  double omega_corr[64];        // omega_k * (1/G - 1)
};

// One warp per cached position, all kv heads; lanes as in rope_prepass_kernel.
template <int D>
__global__ void __launch_bounds__(256) cache_rephase_kernel(const __grid_constant__ RephaseArgs a) {
  constexpr int P = D / 2;
  constexpr int NPAIR = 8;
  constexpr int LANES_PER_ROW = P / NPAIR;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long j_ll = a.j_begin + static_cast<long long>(blockIdx.x) * 8 + warp;
  if (j_ll >= a.P0) return;
  const int j = static_cast<int>(j_ll);
  const int grp = lane >> 3, l8 = lane & 7;
  if (l8 >= LANES_PER_ROW) return;
  const int k0 = l8 * NPAIR;
  float cc[NPAIR], sc[NPAIR];
  if (a.need_long) {
    const double jd = static_cast<double>(j);
    const double jg = static_cast<double>(j / a.G - j);
#pragma unroll
    for (int i = 0; i < NPAIR; ++i)
      angle_cos_sin(a.mode == 0 ? jd * a.omega_corr[k0 + i] : jg * a.omega[k0 + i], cc[i], sc[i]);
  }
  for (int h = grp; h < a.hkv; h += 4) {
    const __nv_bfloat16* src = a.kcache + (static_cast<long long>(j) * a.hkv + h) * D;
    Vec8<__nv_bfloat16> x1, x2;
    x1.load(src + k0);
    x2.load(src + P + k0);
    float u[8], w[8];
#pragma unroll
    for (int i = 0; i < NPAIR; ++i) {
      u[i] = x1.get(i);
      w[i] = x2.get(i);
    }
    bool fin = true;
#pragma unroll
    for (int i = 0; i < NPAIR; ++i) fin &= f16_ok(u[i]) & f16_ok(w[i]);
    __half* dst_o = a.Ko + (static_cast<long long>(h) * a.Lk + j) * D;
    store8_f16(dst_o + k0, u);
    store8_f16(dst_o + P + k0, w);
    if (a.need_long) {
      float y1[8], y2[8];
#pragma unroll
      for (int i = 0; i < NPAIR; ++i) {
        y1[i] = u[i] * cc[i] - w[i] * sc[i];
        y2[i] = w[i] * cc[i] + u[i] * sc[i];
      }
#pragma unroll
      for (int i = 0; i < NPAIR; ++i) fin &= f16_ok(y1[i]) & f16_ok(y2[i]);
      __half* dst_l = a.Kl + (static_cast<long long>(h) * a.Lk + j) * D;
      store8_f16(dst_l + k0, y1);
      store8_f16(dst_l + P + k0, y2);
    }
    if (!fin) report_status(kDevRange, 41);
  }
}

}  // namespace bf
