// Bifocal causal prefill on the warp-level tensor core path (mma.sync m16n8k16).
//
// Operands come from the RoPE pre-pass: Qo/Ql [b, hq, L, D] and Ko/Kl [b, hkv, L, D]
// (original / long-range RoPE, bf16), V [b, L, hkv, D] bf16. Each CTA owns 128 query
// rows of one head (8 warps x 16 rows) and walks the causal key tiles (64 keys) with a
// two-stage cp.async pipeline. Per (query-tile, key-tile) it loads only the key forms
// the tile needs: Ko if some pair is inside the local window (i - j < w0), Kl if some
// pair is outside it. Inside a warp the score of each pair is taken from the branch
// that owns it, and one online softmax runs over the merged row: this is the
// inclusion-exclusion merge of the ai-feeds summary (方法, key module 3) without
// forming the subtracted terms.
#pragma once
#include "common.cuh"

namespace bf {

struct AttnArgs {
  const __half* Qo;  // fp16 QK^T operands from the pre-pass
  const __half* Ql;
  const __half* Ko;
  const __half* Kl;
  const __nv_bfloat16* V;
  long long v_row_stride;    // elements between consecutive positions of V (hkv * D)
  long long v_batch_stride;  // elements between batches of V
  __nv_bfloat16* out;        // [b, L, hq, D]
  float* lse;                // [b, hq, L] or null
  int L, hq, hkv, w0;
  float scale_log2;  // softmax scale * log2(e)
};

namespace mma_cfg {
constexpr int BM = 128;
constexpr int BN = 64;
constexpr int WARPS = 8;
}  // namespace mma_cfg

template <int D>
__device__ __forceinline__ uint32_t swz_off(int row, int chunk) {
  return static_cast<uint32_t>(row * (D * 2) + ((chunk ^ (row & 7)) << 4));
}

// Copy `rows` rows of D bf16 (global row stride `gstride` elements) into a swizzled
// shared tile; rows at or beyond `valid` are zero-filled.
template <int D, int ROWS, typename T>
__device__ __forceinline__ void load_tile_async(uint32_t sbase, const T* g, long long gstride, int valid) {
  constexpr int CH = D / 8;
  for (int idx = threadIdx.x; idx < ROWS * CH; idx += mma_cfg::WARPS * 32) {
    const int r = idx / CH, c = idx % CH;
    const bool ok = r < valid;
    const T* src = g + (ok ? static_cast<long long>(r) * gstride + c * 8 : 0);
    cp_async_16(sbase + swz_off<D>(r, c), src, ok);
  }
}

template <int D, bool BIFOCAL>
__global__ void __launch_bounds__(256, 1) attn_mma_kernel(const __grid_constant__ AttnArgs a) {
  using namespace mma_cfg;
  constexpr int KC = D / 16;  // k-chunks of the QK^T contraction
  constexpr int NT = BN / 8;  // n-tiles of S
  constexpr int DT = D / 8;   // n-tiles of O
  constexpr int NV = BIFOCAL ? 2 : 1;
  constexpr uint32_t QTILE = BM * D * 2, KTILE = BN * D * 2;

  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sQ = smem_u32(smem);                    // [NV][BM][D]
  const uint32_t sK = sQ + NV * QTILE;                   // [2 stages][NV][BN][D]
  const uint32_t sV = sK + 2 * NV * KTILE;               // [2 stages][BN][D]

  const int n_qt = (a.L + BM - 1) / BM;
  const int qt = n_qt - 1 - blockIdx.x;  // heaviest tiles first
  const int h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (a.hq / a.hkv);
  const int i0 = qt * BM;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int w0 = a.w0;

  const long long qoff = (static_cast<long long>(b) * a.hq + h) * a.L * D + static_cast<long long>(i0) * D;
  const long long koff = (static_cast<long long>(b) * a.hkv + kvh) * a.L * D;
  const __nv_bfloat16* Vg = a.V + b * a.v_batch_stride + kvh * D;

  const int qvalid = min(BM, a.L - i0);
  load_tile_async<D, BM>(sQ, a.Qo + qoff, D, qvalid);
  if (BIFOCAL) load_tile_async<D, BM>(sQ + QTILE, a.Ql + qoff, D, qvalid);
  cp_async_commit();

  const int kv_end = min(i0 + BM, a.L);
  const int n_kt = (kv_end + BN - 1) / BN;

  auto tile_needs = [&](int j0, bool& need_o, bool& need_l) {
    if (!BIFOCAL) {
      need_o = true;
      need_l = false;
      return;
    }
    const int dmin = i0 - (j0 + BN - 1), dmax = i0 + BM - 1 - j0;
    need_o = (w0 > 0) && (dmin < w0);
    need_l = dmax >= w0;
  };
  auto issue_kv = [&](int t) {
    const int j0 = t * BN, st = t & 1;
    const int valid = min(BN, a.L - j0);
    bool no, nl;
    tile_needs(j0, no, nl);
    const uint32_t kb = sK + st * NV * KTILE;
    if (no) load_tile_async<D, BN>(kb, a.Ko + koff + static_cast<long long>(j0) * D, D, valid);
    if (BIFOCAL && nl) load_tile_async<D, BN>(kb + KTILE, a.Kl + koff + static_cast<long long>(j0) * D, D, valid);
    load_tile_async<D, BN>(sV + st * KTILE, Vg + static_cast<long long>(j0) * a.v_row_stride, a.v_row_stride, valid);
  };
  issue_kv(0);
  cp_async_commit();

  const int r0 = warp * 16;  // warp's first row inside the tile
  const int iw = i0 + r0;    // warp's first query row
  const int g8 = lane >> 2, t4 = lane & 3;
  float o[DT][4];
#pragma unroll
  for (int i = 0; i < DT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};

  for (int t = 0; t < n_kt; ++t) {
    if (t + 1 < n_kt) issue_kv(t + 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

    const int j0 = t * BN, st = t & 1;
    const int dmin = iw - (j0 + BN - 1), dmax = iw + 15 - j0;
    if (dmax >= 0) {
      bool use_o = true, use_l = false;
      if (BIFOCAL) {
        use_o = (w0 > 0) && (dmin < w0);
        use_l = dmax >= w0;
      }
      float s[NT][4];
#pragma unroll
      for (int i = 0; i < NT; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
      const uint32_t kb = sK + st * NV * KTILE;
      // S over one branch: variant v of Q against variant v of K
      auto qk = [&](int v, float (&acc)[NT][4]) {
#pragma unroll
        for (int kc = 0; kc < KC; ++kc) {
          uint32_t af[4];
          ldmatrix_x4(af, sQ + v * QTILE + swz_off<D>(r0 + (lane & 15), 2 * kc + (lane >> 4)));
#pragma unroll
          for (int nt = 0; nt < NT; nt += 2) {
            uint32_t bfr[4];
            const int krow = nt * 8 + (lane & 7) + ((lane >> 4) << 3);
            ldmatrix_x4(bfr, kb + v * KTILE + swz_off<D>(krow, 2 * kc + ((lane >> 3) & 1)));
            mma_f16_16816(acc[nt], af, bfr[0], bfr[1]);
            mma_f16_16816(acc[nt + 1], af, bfr[2], bfr[3]);
          }
        }
      };
      if (use_o) qk(0, s);
      if (BIFOCAL && use_l) {
        if (!use_o) {
          qk(1, s);
        } else {
          float sl[NT][4];
#pragma unroll
          for (int i = 0; i < NT; ++i) sl[i][0] = sl[i][1] = sl[i][2] = sl[i][3] = 0.f;
          qk(1, sl);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = iw + g8 + ((e >> 1) << 3);
              const int j = j0 + nt * 8 + 2 * t4 + (e & 1);
              if (i - j >= w0) s[nt][e] = sl[nt][e];
            }
        }
      }
      // scale into the log2 domain, causal mask, online softmax
      const bool need_mask = dmin < 0;
      float mx[2] = {m_r[0], m_r[1]};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float x = s[nt][e] * a.scale_log2;
          if (need_mask) {
            const int i = iw + g8 + ((e >> 1) << 3);
            const int j = j0 + nt * 8 + 2 * t4 + (e & 1);
            if (j > i) x = -INFINITY;
          }
          s[nt][e] = x;
          mx[e >> 1] = fmaxf(mx[e >> 1], x);
        }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      }
      float alpha[2], ref[2], rs[2] = {0.f, 0.f};
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        ref[r] = (mx[r] == -INFINITY) ? 0.f : mx[r];
        alpha[r] = fast_exp2(m_r[r] - ref[r]);
        m_r[r] = mx[r];
      }
      uint32_t pa[NT / 2][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float p0 = fast_exp2(s[nt][0] - ref[0]), p1 = fast_exp2(s[nt][1] - ref[0]);
        const float p2 = fast_exp2(s[nt][2] - ref[1]), p3 = fast_exp2(s[nt][3] - ref[1]);
        rs[0] += p0 + p1;
        rs[1] += p2 + p3;
        const int kk = nt >> 1, hi = nt & 1;
        pa[kk][hi * 2 + 0] = pack_bf16x2(p0, p1);
        pa[kk][hi * 2 + 1] = pack_bf16x2(p2, p3);
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) l_r[r] = l_r[r] * alpha[r] + rs[r];
#pragma unroll
      for (int dt = 0; dt < DT; ++dt) {
        o[dt][0] *= alpha[0];
        o[dt][1] *= alpha[0];
        o[dt][2] *= alpha[1];
        o[dt][3] *= alpha[1];
      }
      // O += P V
      const uint32_t vb = sV + st * KTILE;
#pragma unroll
      for (int kk = 0; kk < BN / 16; ++kk) {
        const uint32_t af[4] = {pa[kk][0], pa[kk][1], pa[kk][2], pa[kk][3]};
#pragma unroll
        for (int dt = 0; dt < DT; dt += 2) {
          uint32_t bfr[4];
          const int vrow = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
          ldmatrix_x4_trans(bfr, vb + swz_off<D>(vrow, dt + (lane >> 4)));
          mma_bf16_16816(o[dt], af, bfr[0], bfr[1]);
          mma_bf16_16816(o[dt + 1], af, bfr[2], bfr[3]);
        }
      }
    }
    __syncthreads();
  }

  // epilogue: rows g8 and g8 + 8 of this warp
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    float lsum = l_r[r];
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
    const int i = iw + g8 + r * 8;
    if (i < a.L) {
      const float inv = 1.f / lsum;
      __nv_bfloat16* orow = a.out + ((static_cast<long long>(b) * a.L + i) * a.hq + h) * D;
#pragma unroll
      for (int dt = 0; dt < DT; ++dt) {
        const uint32_t pk = pack_bf16x2(o[dt][2 * r] * inv, o[dt][2 * r + 1] * inv);
        *reinterpret_cast<uint32_t*>(orow + dt * 8 + 2 * t4) = pk;
      }
      if (a.lse && t4 == 0)
        a.lse[(static_cast<long long>(b) * a.hq + h) * a.L + i] = (m_r[r] + __log2f(lsum)) * 0.69314718055994530942f;
    }
  }
}

template <int D, bool BIFOCAL>
constexpr int attn_mma_smem_bytes() {
  return (BIFOCAL ? 2 : 1) * mma_cfg::BM * D * 2 + 2 * (BIFOCAL ? 2 : 1) * mma_cfg::BN * D * 2 +
         2 * mma_cfg::BN * D * 2;
}

}  // namespace bf
