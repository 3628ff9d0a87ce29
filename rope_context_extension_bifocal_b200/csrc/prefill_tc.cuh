// Bifocal causal prefill on the 5th-generation tensor cores (tcgen05 + TMEM + TMA), D = 128.
//
// One CTA owns 128 query rows of one head. Tensor memory (512 columns) holds
//   [  0,  64) Q under the original RoPE   (fp16, the A operand of QK^T)
//   [ 64, 128) Q under the long-range RoPE  (fp16)
//   [128, 256) S buffer 0 / P buffer 0       (S fp32; P bf16 written over its first 64 columns)
//   [256, 384) S buffer 1 / P buffer 1
//   [384, 512) O accumulator (fp32)
// so both GEMMs read only their B operand (a K or V tile) from shared memory. K and V
// tiles (128 keys x 128 d) arrive by TMA into a ring of 32 KB slots.
//
// Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer (one thread), warps 2..9 =
// softmax. A softmax thread owns one query row and one half of the 128 key columns (warp w
// reads TMEM lanes 32*(w%4).., warps 2-5 the left half, 6-9 the right half); the two halves
// of a row exchange their maxima through shared memory. Per key tile the MMA warp issues
// S = Q K^T into the free S buffer while the softmax works on the other one, then
// O += P V once the softmax has published P.
//
// Bifocal structure (ai-feeds summary of Jet-Long, 方法 key modules 1 and 3): a key tile
// whose pairs all lie inside the local window (i - j < w0) is scored with the original
// RoPE forms, one whose pairs all lie outside with the long-range forms; a tile the band
// edge crosses is visited twice, once per branch, each visit masking the pairs the other
// branch owns. One online softmax runs over all visits, which is the inclusion-exclusion
// merge without forming the subtracted terms.
#pragma once
#include "common.cuh"

namespace bf {
namespace tc {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int D = 128;
constexpr int NSLOT = 6;
constexpr uint32_t SLOT_BYTES = 32768;  // one K or V tile: two 128-row x 128-byte swizzled halves
constexpr uint32_t HALF_BYTES = 16384;
constexpr int NTHREADS = 320;  // 10 warps: TMA, MMA, 8 softmax (two per TMEM lane quadrant)
constexpr uint32_t COL_QO = 0, COL_QL = 64, COL_S = 128, COL_O = 384, NCOLS = 512;
constexpr float RESCALE_THRESHOLD = 8.f;  // log2 units: O is rescaled only when the row max grows by more

enum VKind : int { ORIG_FULL = 0, LONG_FULL = 1, ORIG_LOCAL = 2, LONG_ONLY = 3 };

// instruction descriptors (kind::f16): D f32, M = 128, N = 128
constexpr uint32_t IDESC_QK = (1u << 4) | (0u << 7) | (0u << 10) | (16u << 17) | (8u << 24);  // f16 x f16, K-major
constexpr uint32_t IDESC_PV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | (16u << 17) | (8u << 24);  // bf16, B MN-major

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// K tile (K-major, 128B swizzle): k-step kk (16 elements) of 8
__device__ __forceinline__ uint64_t k_desc(uint32_t slot, int kk) {
  return smem_desc(slot + (kk >> 2) * HALF_BYTES + (kk & 3) * 32, 16, 1024);
}
// V tile (MN-major, 128B swizzle): k-step kk covers keys 16kk .. 16kk+15; the two
// 64-wide d halves are 16 KB apart
__device__ __forceinline__ uint64_t v_desc(uint32_t slot, int kk) {
  return smem_desc(slot + kk * 2048, HALF_BYTES, 1024);
}

__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n"
      "}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 consecutive TMEM columns of this thread's lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]));
}

}  // namespace tc

struct TcArgs {
  CUtensorMap ko_map;  // fp16 [b*hkv][L][128], box (64, 128, 1), 128B swizzle
  CUtensorMap kl_map;
  CUtensorMap v_map;   // bf16 [b][L][hkv][128], box (64, 1, 128, 1), 128B swizzle
  const __half* Qo;    // [b, hq, L, 128]
  const __half* Ql;
  __nv_bfloat16* out;  // [b, L, hq, 128]
  float* lse;          // [b, hq, L] or null
  int L, hq, hkv, batch, w0;
  float scale_log2;
};

// Visits of key tile t for the query tile starting at i0: kinds (and how many, 1 or 2).
template <bool BIFOCAL>
__device__ __forceinline__ int tile_visits(int i0, int t, int w0, int (&kinds)[2]) {
  if (!BIFOCAL) {
    kinds[0] = tc::ORIG_FULL;
    return 1;
  }
  const int j0 = t * tc::BN;
  const int dmin = i0 - (j0 + tc::BN - 1), dmax = i0 + tc::BM - 1 - j0;
  if (dmin >= w0) {
    kinds[0] = tc::LONG_FULL;
    return 1;
  }
  if (dmax < w0) {
    kinds[0] = tc::ORIG_FULL;
    return 1;
  }
  if (w0 > 0) {
    kinds[0] = tc::ORIG_LOCAL;
    kinds[1] = tc::LONG_ONLY;
    return 2;
  }
  kinds[0] = tc::LONG_ONLY;
  return 1;
}

template <bool BIFOCAL>
__global__ void __launch_bounds__(tc::NTHREADS, 1) attn_tc_kernel(const __grid_constant__ TcArgs a) {
  using namespace tc;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ uint64_t full[NSLOT], empty[NSLOT], s_full[2], p_ready[2], o_done, q_ready, mma_drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int s_abort;
  __shared__ float red[2][2][BM];  // [visit parity][column half][row]: row maxima, then row sums

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = (a.L + BM - 1) / BM;
  const int per_tile = a.hq * a.batch;
  const int qt = n_qt - 1 - static_cast<int>(blockIdx.x) / per_tile;  // heaviest first
  const int rem = static_cast<int>(blockIdx.x) % per_tile;
  const int h = rem % a.hq, b = rem / a.hq;
  const int kvh = h / (a.hq / a.hkv);
  const int i0 = qt * BM;
  const int n_kt = (min(i0 + BM, a.L) + BN - 1) / BN;
  const uint32_t slots = smem_u32(smem);

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_ready[i], 8);
    }
    mbar_init(&o_done, 1);
    mbar_init(&q_ready, 8);
    mbar_init(&mma_drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                 "r"(NCOLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&a.ko_map);
      if (BIFOCAL) prefetch_tensormap(&a.kl_map);
      prefetch_tensormap(&a.v_map);
      int n = 0;  // slot fills issued
      const int krow = b * a.hkv + kvh;
      bool ok = true;
      for (int t = 0; t < n_kt && ok; ++t) {
        int kinds[2];
        const int nv = tile_visits<BIFOCAL>(i0, t, a.w0, kinds);
        for (int vi = 0; vi < nv && ok; ++vi) {
          const bool lng = kinds[vi] == LONG_FULL || kinds[vi] == LONG_ONLY;
          for (int x = 0; x < 2 && ok; ++x, ++n) {
            const int slot = n % NSLOT, use = n / NSLOT;
            if (use > 0 && !mbar_wait_abortable(&empty[slot], (use - 1) & 1, 10, &s_abort)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[slot], SLOT_BYTES);
            uint8_t* dst = smem + slot * SLOT_BYTES;
            if (x == 0) {
              const CUtensorMap* m = lng ? &a.kl_map : &a.ko_map;
              tma_load_3d(dst, m, &full[slot], 0, t * BN, krow);
              tma_load_3d(dst + HALF_BYTES, m, &full[slot], 64, t * BN, krow);
            } else {
              tma_load_4d(dst, &a.v_map, &full[slot], 0, kvh, t * BN, b);
              tma_load_4d(dst + HALF_BYTES, &a.v_map, &full[slot], 64, kvh, t * BN, b);
            }
          }
        }
      }
      // drain: every fill issued must have landed before the CTA may exit
      const int first = n > NSLOT ? n - NSLOT : 0;
      for (int k = first; k < n; ++k) mbar_wait(&full[k % NSLOT], (k / NSLOT) & 1, 11);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait_abortable(&q_ready, 0, 20, &s_abort);
      fence_after();
      int v = 0;  // visit index
      int prev_vslot = -1;
      for (int t = 0; t < n_kt && ok; ++t) {
        int kinds[2];
        const int nv = tile_visits<BIFOCAL>(i0, t, a.w0, kinds);
        for (int vi = 0; vi < nv && ok; ++vi, ++v) {
          const bool lng = kinds[vi] == LONG_FULL || kinds[vi] == LONG_ONLY;
          const int ks = (2 * v) % NSLOT, vs = (2 * v + 1) % NSLOT;
          // S(v) = Q K^T into S buffer v % 2
          if (!mbar_wait_abortable(&full[ks], ((2 * v) / NSLOT) & 1, 21, &s_abort)) {
            ok = false;
            break;
          }
          fence_after();
          const uint32_t s_col = tmem + COL_S + (v & 1) * 128;
          const uint32_t q_col = tmem + (lng ? COL_QL : COL_QO);
          const uint32_t kslot = slots + ks * SLOT_BYTES;
          // descriptors formed once per group: tcgen05.mma issue waits on the previous MMA, so
          // arithmetic between the K-steps would stretch the group
          const uint64_t kd0 = k_desc(kslot, 0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(s_col, q_col + kk * 8, kd0 + (((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4), IDESC_QK, kk > 0);
          mma_commit(&s_full[v & 1]);
          mma_commit(&empty[ks]);
          // O += P(v-1) V(v-1)
          if (v >= 1) {
            if (!mbar_wait_abortable(&p_ready[(v - 1) & 1], ((v - 1) >> 1) & 1, 22, &s_abort) ||
                !mbar_wait_abortable(&full[prev_vslot], ((2 * (v - 1) + 1) / NSLOT) & 1, 23, &s_abort)) {
              ok = false;
              break;
            }
            fence_after();
            const uint32_t p_col = tmem + COL_S + ((v - 1) & 1) * 128;
            const uint32_t vslot = slots + prev_vslot * SLOT_BYTES;
            const uint64_t vd0 = v_desc(vslot, 0);
            const uint32_t acc0 = v - 1 > 0;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ts(tmem + COL_O, p_col + kk * 8, vd0 + kk * (2048 >> 4), IDESC_PV, kk > 0 ? 1u : acc0);
            mma_commit(&empty[prev_vslot]);
            mma_commit(&o_done);
          }
          prev_vslot = vs;
        }
      }
      // last visit's PV
      if (ok && v >= 1) {
        if (mbar_wait_abortable(&p_ready[(v - 1) & 1], ((v - 1) >> 1) & 1, 24, &s_abort) &&
            mbar_wait_abortable(&full[prev_vslot], ((2 * (v - 1) + 1) / NSLOT) & 1, 25, &s_abort)) {
          fence_after();
          const uint32_t p_col = tmem + COL_S + ((v - 1) & 1) * 128;
          const uint32_t vslot = slots + prev_vslot * SLOT_BYTES;
          const uint64_t vd0 = v_desc(vslot, 0);
          const uint32_t acc0 = v - 1 > 0;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + COL_O, p_col + kk * 8, vd0 + kk * (2048 >> 4), IDESC_PV, kk > 0 ? 1u : acc0);
          mma_commit(&empty[prev_vslot]);
          mma_commit(&o_done);
        }
      }
      // every MMA issued has finished before teardown
      mma_commit(&mma_drain);
      mbar_wait(&mma_drain, 0, 26);
    }
  } else {
    // ------------------------------------------------------------ softmax warps 2..9
    const int quad = warp & 3;          // TMEM lane quadrant this warp may access
    const int half = (warp - 2) >> 2;   // which 64 of the 128 key columns
    const int r = quad * 32 + lane;     // row within the tile
    const int i = i0 + r;               // query row
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t bar_id = 1 + quad;   // named barrier of the two warps sharing these rows
    // Q (both RoPE forms) into TMEM: lane = row, 64 columns of fp16 pairs each; each half
    // of the row's threads writes 32 columns of each form
    {
      const long long qrow = ((static_cast<long long>(b) * a.hq + h) * a.L + i) * D;
      for (int f = 0; f < (BIFOCAL ? 2 : 1); ++f) {
        const __half* src = (f == 0 ? a.Qo : a.Ql) + qrow;
        const int c0 = 32 * half;
        uint32_t reg[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          uint4 x = make_uint4(0u, 0u, 0u, 0u);
          if (i < a.L) x = reinterpret_cast<const uint4*>(src)[c0 / 4 + u];
          reg[4 * u + 0] = x.x;
          reg[4 * u + 1] = x.y;
          reg[4 * u + 2] = x.z;
          reg[4 * u + 3] = x.w;
        }
        tmem_st32(lane_addr + (f == 0 ? COL_QO : COL_QL) + c0, reg);
      }
      wait_st();
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&q_ready);
    }

    // After an expired wait (ok == false, warp-uniform) a warp does no more work but still
    // passes every named barrier its partner warp passes, so the pair cannot deadlock.
    float m_ref = -INFINITY, l_half = 0.f;
    int v = 0;
    bool ok = true;
    for (int t = 0; t < n_kt; ++t) {
      int kinds[2];
      const int nv = tile_visits<BIFOCAL>(i0, t, a.w0, kinds);
      const int j0 = t * BN;
      for (int vi = 0; vi < nv; ++vi, ++v) {
        const int kind = kinds[vi];
        // every lane waits; the result is made warp-uniform because the TMEM accesses
        // below are warp-collective (.sync.aligned)
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait_abortable(&s_full[v & 1], (v >> 1) & 1, 30, &s_abort));
        const uint32_t s_addr = lane_addr + COL_S + (v & 1) * 128;
        float s[64];
        float mh = -INFINITY;
        if (ok) {
          fence_after();
          tmem_ld32(s_addr + 64 * half, s);
          tmem_ld32(s_addr + 64 * half + 32, s + 32);
          wait_ld();
          // mask (only on visits that need one)
          const bool masked = kind != LONG_FULL && (kind != ORIG_FULL || j0 + BN - 1 > i0);
          if (masked) {
            const int d0 = i - j0 - 64 * half;  // i - j for this thread's first column
            const int lo = (kind == LONG_ONLY) ? a.w0 : 0;            // keep lo <= i - j
            const int hi = (kind == ORIG_LOCAL) ? a.w0 : 0x7fffffff;  //      and i - j < hi
#pragma unroll
            for (int c = 0; c < 64; ++c) {
              const int d = d0 - c;
              s[c] = (d >= lo && d < hi) ? s[c] : -INFINITY;
            }
          }
          // raw max of this half with independent accumulators
          float m8[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) m8[u] = s[u];
#pragma unroll
          for (int c = 8; c < 64; c += 8)
#pragma unroll
            for (int u = 0; u < 8; ++u) m8[u] = fmaxf(m8[u], s[c + u]);
          mh = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
        }
        // the row max with the other half
        red[v & 1][half][r] = mh;
        asm volatile("bar.sync %0, 64;" ::"r"(bar_id) : "memory");
        mh = fmaxf(mh, red[v & 1][half ^ 1][r]);
        if (ok) {
          const float mx = mh * a.scale_log2;  // scale > 0: max commutes with it
          // lazy rescale (both halves take the same decision): a row keeps its reference
          // unless its max grew by more than the threshold
          float alpha = 1.f;
          bool grow = false;
          if (mx > m_ref + RESCALE_THRESHOLD || (m_ref == -INFINITY && mx > -INFINITY)) {
            alpha = (m_ref == -INFINITY) ? 0.f : fast_exp2(m_ref - mx);
            grow = m_ref != -INFINITY;  // O already holds this row's earlier terms
            m_ref = mx;
          }
          const float neg_ref = (m_ref == -INFINITY) ? 0.f : -m_ref;
          const float sc = a.scale_log2;
          float r8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            const float p0 = fast_exp2(fmaf(s[c], sc, neg_ref)), p1 = fast_exp2(fmaf(s[c + 1], sc, neg_ref));
            r8[(c >> 1) & 7] += p0 + p1;
            pk[c >> 1] = pack_bf16x2(p0, p1);
          }
          const float rs = ((r8[0] + r8[1]) + (r8[2] + r8[3])) + ((r8[4] + r8[5]) + (r8[6] + r8[7]));
          l_half = l_half * alpha + rs;
          tmem_st32(s_addr + 32 * half, pk);  // P (bf16 pairs) over the first 64 columns of the S buffer
          // O must hold PV(v-1) before it is rescaled and before PV(v) adds to it
          if (v >= 1) ok = __all_sync(0xffffffffu, mbar_wait_abortable(&o_done, (v - 1) & 1, 31, &s_abort));
          if (ok && v >= 1) {
            fence_after();
            // warp-uniform: rescale this half of O if any row of the warp needs it (others scale by 1)
            if (__any_sync(0xffffffffu, grow)) {
              const float f = grow ? alpha : 1.f;
              const uint32_t o_addr = lane_addr + COL_O + 64 * half;
#pragma unroll 1
              for (int c = 0; c < 64; c += 32) {
                float ov[32];
                tmem_ld32(o_addr + c, ov);
                wait_ld();
                uint32_t ou[32];
#pragma unroll
                for (int u = 0; u < 32; ++u) ou[u] = __float_as_uint(ov[u] * f);
                tmem_st32(o_addr + c, ou);
              }
            }
          }
          wait_st();
          fence_before();
          __syncwarp();
          if (ok && lane == 0) mbar_arrive(&p_ready[v & 1]);
        }
      }
    }
    // epilogue: row sum of both halves, O / l -> bf16 (each half its 64 columns), LSE
    const bool fin = ok && v >= 1 && __all_sync(0xffffffffu, mbar_wait_abortable(&o_done, (v - 1) & 1, 32, &s_abort));
    red[0][half][r] = l_half;
    asm volatile("bar.sync %0, 64;" ::"r"(bar_id) : "memory");
    const float l_sum = l_half + red[0][half ^ 1][r];
    if (fin) {
      fence_after();
      const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
      __nv_bfloat16* orow = a.out + ((static_cast<long long>(b) * a.L + i) * a.hq + h) * D + 64 * half;
#pragma unroll 1
      for (int c = 0; c < 64; c += 32) {
        float ov[32];
        tmem_ld32(lane_addr + COL_O + 64 * half + c, ov);
        wait_ld();
        if (i < a.L) {
#pragma unroll
          for (int u = 0; u < 32; u += 8) {
            uint4 w;
            w.x = pack_bf16x2(ov[u] * inv, ov[u + 1] * inv);
            w.y = pack_bf16x2(ov[u + 2] * inv, ov[u + 3] * inv);
            w.z = pack_bf16x2(ov[u + 4] * inv, ov[u + 5] * inv);
            w.w = pack_bf16x2(ov[u + 6] * inv, ov[u + 7] * inv);
            *reinterpret_cast<uint4*>(orow + c + u) = w;
          }
        }
      }
      if (half == 0 && a.lse && i < a.L)
        a.lse[(static_cast<long long>(b) * a.hq + h) * a.L + i] = (m_ref + __log2f(l_sum)) * 0.69314718055994530942f;
    }
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(NCOLS));
}

constexpr int attn_tc_smem_bytes() { return tc::NSLOT * tc::SLOT_BYTES; }

}  // namespace bf
