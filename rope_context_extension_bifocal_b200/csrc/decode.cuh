// Single-batch decode: append, split-KV partial attention, log-sum-exp combine.
//
// The cache holds keys under the ORIGINAL RoPE (bf16). A cached key j that falls in
// the long-range branch (p - j >= w0) is re-phased on the fly by the correction
// rotation Rcorr(j) = R_long(j) R_orig(j)^-1, whose angle for pair k is
//   j * omega_k * (1/G - 1)          (frequency interpolation)
//   (floor(j / G) - j) * omega_k     (position aliasing)
// (ai-feeds summary of Jet-Long, 方法 key module 3: the correction rotation of cached
// keys; knowledge-base note, 设计原理: the near/far boundary slides during generation).
// The rotation runs in registers on tiles staged in shared memory by TMA, so the cache
// is read once from HBM and never rewritten. G follows the current length L, so when
// L crosses a multiple of w_pretrained every long-range key is re-phased at once.
//
// Work split: CTA = (key range, up to 4 kv heads). A TMA warp streams 16-key stages
// (K and V, every head, both 64-element halves of D) through a 5-deep mbarrier ring, two
// table warps build each stage's correction cos/sin table; two consumer warps per kv head each take
// one 8-key n-tile of every stage, keeping their own online softmax, and merge the two states in
// shared memory at the end, so each key range leaves one partial per query head. QK^T of the
// g = hq/hkv query rows runs on mma.sync m16n8k16 (rows in M); PV runs transposed,
// O^T = V^T P^T on m16n8k8, so the query rows sit in N and the accumulator is D x 8.
// QK^T operands are fp16 (rotated query, corrected or converted cached key), PV is bf16.
#pragma once
#include "common.cuh"

namespace bf {

namespace dec {
constexpr int KB = 16;      // keys per stage
constexpr int NST = 5;      // stages in the ring (4 in flight while one is consumed)
constexpr int HPC = 4;      // kv heads per CTA (max)
constexpr int MAX_G = 8;    // query heads per kv head (max)
}  // namespace dec

struct DecodeArgs {
  CUtensorMap kmap;  // cache K viewed as (d_lo 64, d_hi D/64, head hkv, key cap), box (64,1,1,KB)
  CUtensorMap vmap;
  const __nv_bfloat16* q;  // [hq, D] raw
  float* part_o;           // [n_split, hq, D] unnormalised (batched: parts_stride rows per sequence)
  float* part_ml;          // [n_split, hq, 2]: running max (log2 domain), sum
  int L, hq, hkv, w0, G, mode, bifocal;
  int key0;  // first key read: 0, or L - w0 for a sliding window
  int split_len, n_split;
  float scale_log2;
  double omega[64];
  double omega_long[64];  // omega / G
  double omega_corr[64];  // omega * (1/G - 1)
  // Batched form over a paged cache (grid.z = sequence; null seq_lens = the single call above):
  // sequence b has length seq_lens[b] (with its new token); its logical key j lives in pool
  // row block_table[b * max_pages + j / page_size] * page_size + j % page_size. G, the band
  // edge and the long-range tables follow each sequence's own length.
  const int* seq_lens;
  const int* block_table;
  int max_pages, page_size, w_pretrained, force_bifocal;
  int pool_pages;    // block-table entries must lie in [0, pool_pages); lengths in [1, L = max_len]
  int parts_stride;  // partial rows reserved per sequence
  int test_skip_stage;  // test only (bifocal_test_set_fault): 1 + the stage CTA 0's producer never issues; 0 = off
};

// 128-byte swizzle of TMA SWIZZLE_128B: 16-byte chunk c of row r sits at chunk c ^ (r & 7).
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// TEST = true is the instantiation launched only while bifocal_test_set_fault has armed a
// skipped stage: its producer stops issuing at that stage in CTA 0. The normal instantiation has
// no trace of it (a changed loop bound in the producer cost up to 20 us per step).
// Correction rotation of two pairs held as bf16x2 (x = elements d, d+1; y = elements d+P,
// d+P+1) by {cos d, cos d+1, sin d, sin d+1}, on packed fp32 pairs; the result as fp16x2.
__device__ __forceinline__ uint32_t rot_x(uint32_t x, uint32_t y, float4 cs) {
  const uint64_t X = bf16x2_to_f2(x), Y = bf16x2_to_f2(y);
  return f2_to_f16x2(f2_sub(f2_mul(X, f2_pack(cs.x, cs.y)), f2_mul(Y, f2_pack(cs.z, cs.w))));
}
__device__ __forceinline__ uint32_t rot_y(uint32_t x, uint32_t y, float4 cs) {
  const uint64_t X = bf16x2_to_f2(x), Y = bf16x2_to_f2(y);
  return f2_to_f16x2(f2_fma(X, f2_pack(cs.z, cs.w), f2_mul(Y, f2_pack(cs.x, cs.y))));
}

template <int D, bool TEST>
__global__ void __launch_bounds__((2 * dec::HPC + 3) * 32, 1) decode_partial_kernel(const __grid_constant__ DecodeArgs a) {
  using namespace dec;
  constexpr int P = D / 2;
  constexpr int HALVES = D / 64;
  constexpr int KC = D / 16;       // k-chunks of QK^T
  constexpr int KCP = KC / 2;      // k-chunks holding the first element of each pair
  constexpr int MT = D / 16;       // m-tiles of O^T (16 d-values each)
  constexpr uint32_t HEAD_TILE = KB * 128;                 // one head, one half: KB rows x 128 B
  constexpr uint32_t STAGE_KV = HPC * HALVES * HEAD_TILE;  // all heads, all halves (K or V)
  constexpr int CS_STRIDE = P * 8 + 64;  // bytes per key row of the cos/sin table (pad: rows 16 banks apart)
  constexpr uint32_t STAGE_CS = KB * CS_STRIDE;

  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sK = smem;                       // [NST][HPC][HALVES][KB][128 B]
  uint8_t* sV = sK + NST * STAGE_KV;        // same
  uint8_t* sCS = sV + NST * STAGE_KV;       // [NST][KB][CS_STRIDE]: correction cos/sin per stage
  // full[s]: the stage's K/V bytes have landed (producer's expect_tx); tbl[s]: its cos/sin table is
  // written (one arrive per table-warp lane); empty[s]: every consumer warp is done with the slot
  uint64_t* full = reinterpret_cast<uint64_t*>(sCS + NST * STAGE_CS);
  uint64_t* empty = full + NST;
  uint64_t* tbl = empty + NST;
  uint8_t* xch = reinterpret_cast<uint8_t*>(tbl + NST);  // [HPC][4 * MT + 2][32] floats: warp-pair exchange
  __shared__ int s_abort;  // set when a bounded wait expires: later waits return at once

  pdl_launch_dependents();  // the combine may start its prologue; it waits for this grid's writes
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head0 = blockIdx.y * HPC;
  const int nheads = min(HPC, a.hkv - head0);
  const int g = a.hq / a.hkv;
  const bool paged = a.seq_lens != nullptr;
  const int bz = paged ? static_cast<int>(blockIdx.z) : 0;
  const int L = paged ? a.seq_lens[bz] : a.L;
  if (paged && (L < 1 || L > a.L)) {  // a length the batch's tables and partial rows cannot hold (a.L = max_len)
    if (threadIdx.x == 0) report_status(kDevIndex, 52);
    return;
  }
  const int G = paged ? (L <= a.w_pretrained ? 1 : (L + a.w_pretrained - 1) / a.w_pretrained) : a.G;
  const bool bifocal = paged ? (a.force_bifocal || (G > 1 && a.w0 < L)) : (a.bifocal != 0);
  const int p = L - 1;
  const int jbeg = a.key0 + blockIdx.x * a.split_len;
  if (jbeg >= L) return;  // a shorter sequence of the batch: no keys in this split (the combine skips it)
  const int jend = min(L, jbeg + a.split_len);
  const int nstage = (jend - jbeg + KB - 1) / KB;
  const int local_from = bifocal ? max(0, L - a.w0) : 0;  // keys j >= local_from are local
  // long-range tables: the host's for a single call, the same fp64 expressions per sequence when batched
  auto omega_long = [&](int k) { return paged ? a.omega[k] / G : a.omega_long[k]; };
  auto omega_corr = [&](int k) { return paged ? a.omega[k] / G - a.omega[k] : a.omega_corr[k]; };
  const int nconsumers = 2 * nheads;  // two warps per kv head, one 8-key n-tile of each stage each

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&tbl[s], 32);
      mbar_init(&empty[s], nconsumers);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == 2 * HPC) {
    // ---------------- TMA warp: one elected lane streams K/V stages
    if (lane == 0) {
      prefetch_tensormap(&a.kmap);
      prefetch_tensormap(&a.vmap);
      const uint32_t bytes = 2u * nheads * HALVES * HEAD_TILE;
      // test instantiation only: CTA 0 issues no stage from test_skip_stage - 1 on
      const int n_issue = (TEST && (blockIdx.x | blockIdx.y | blockIdx.z) == 0) ? min(nstage, a.test_skip_stage - 1)
                                                                                 : nstage;
      uint32_t used = 0, par = 0;  // per slot: has a fill been issued, parity of the fills issued
      // paged: the block-table entry of the current page and, loaded one page ahead, of the next
      // (the stages of a split walk its pages in order, so the load has a page of stages to land).
      // The page index and the offset in it advance by KB keys per stage without a division.
      const int* trow = a.block_table + static_cast<long long>(bz) * a.max_pages;
      int cur_idx = paged ? jbeg / a.page_size : 0;
      int cur_off = paged ? jbeg - cur_idx * a.page_size : 0;
      int cur_row0 = 0;
      bool new_page = true;
      int nxt_pg = paged ? trow[cur_idx] : 0;
      for (int s = 0; s < n_issue; ++s) {
        const int st = s % NST;
        if (s >= NST && !mbar_wait_abortable(&empty[st], ((s / NST) - 1) & 1, 1, &s_abort)) break;
        const int j0 = jbeg + s * KB;
        // Only row p (the new token) comes from the append kernel; every other row was in the
        // cache before this step, so only the stage holding p waits for that grid.
        if (j0 + KB > p) pdl_wait();
        // pool row of logical key j0 (pages hold a multiple of KB keys, so a stage is one page's)
        int row = j0;
        if (paged) {
          if (new_page) {
            const int pg = nxt_pg;
            nxt_pg = cur_idx + 1 < a.max_pages ? trow[cur_idx + 1] : 0;
            const bool pg_ok = pg >= 0 && pg < a.pool_pages;
            if (!pg_ok) report_status(kDevIndex, 53);
            // a bad entry loads stages that start just past the pool's last row: TMA fills them with zeros
            cur_row0 = pg_ok ? pg * a.page_size : a.pool_pages * a.page_size - cur_off;
            new_page = false;
          }
          row = cur_row0 + cur_off;
          cur_off += KB;
          if (cur_off == a.page_size) {  // pages hold a multiple of KB keys
            cur_off = 0;
            ++cur_idx;
            new_page = true;
          }
        }
        mbar_arrive_expect_tx(&full[st], bytes);
        for (int hh = 0; hh < nheads; ++hh)
          for (int hf = 0; hf < HALVES; ++hf) {
            const uint32_t off = st * STAGE_KV + (hh * HALVES + hf) * HEAD_TILE;
            tma_load_4d(sK + off, &a.kmap, &full[st], 0, hf, head0 + hh, row);
            tma_load_4d(sV + off, &a.vmap, &full[st], 0, hf, head0 + hh, row);
          }
        used |= 1u << st;
        par ^= 1u << st;
      }
      // Every copy issued must land before the CTA exits. The consumers wait for every stage
      // they read, so normally nothing is in flight when they finish and the producer leaves at
      // once (holding this warp until the consumers were done cost 2-6 us per decode step). If a
      // wait expired before the producer got here, it waits (bounded) for the last copy it issued
      // into each slot. An expiry after it left can only come from a copy that did not land
      // within the limit, which no wait could repair.
      if (*reinterpret_cast<volatile int*>(&s_abort))
        for (int st = 0; st < NST; ++st)
          if (used & (1u << st)) mbar_wait_sleepy(&full[st], ((par >> st) & 1u) ^ 1u, 4);
    }
    return;
  }
  if (warp > 2 * HPC) {
    // ---------------- table warps (two, alternating stages): correction cos/sin per (key, pair).
    // Each lane runs 4 chains (pairs 2 lane and 2 lane + 1, keys 0-7 and 8-15 of the stage): an
    // exact angle at the chain's first key, then per-key steps: frequency interpolation adds
    // omega_corr; position aliasing adds -omega unless the next key starts a group of G. A key
    // row holds, per two pairs d, d + 1 (d even), {cos d, cos d+1, sin d, sin d+1}: the consumers'
    // packed fp32 pairs.
    const int cw = warp - 2 * HPC - 1;  // 0 or 1
    const bool lane_on = 2 * lane < P;
    float fi_c[2], fi_s[2], pa_c[2], pa_s[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int pr = 2 * lane + e;
      fi_c[e] = pa_c[e] = 1.f;
      fi_s[e] = pa_s[e] = 0.f;
      if (lane_on) {
        angle_cos_sin(omega_corr(pr), fi_c[e], fi_s[e]);
        angle_cos_sin(-a.omega[pr], pa_c[e], pa_s[e]);
      }
    }
    for (int s = cw; s < nstage; s += 2) {
      const int st = s % NST;
      if (s >= NST && !__all_sync(0xffffffffu, mbar_wait_abortable(&empty[st], ((s / NST) - 1) & 1, 3, &s_abort)))
        break;
      const int j0 = jbeg + s * KB;
      if (j0 < local_from && lane_on) {  // some key of this stage is long-range
        uint8_t* cs = sCS + st * STAGE_CS;
        float c[2][2], sn[2][2];  // [pair 2 lane + e][chain hk]
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
          for (int hk = 0; hk < 2; ++hk) {
            const int pr = 2 * lane + e;
            const int jc = j0 + 8 * hk;
            const double ang0 = (a.mode == 0) ? static_cast<double>(jc) * omega_corr(pr)
                                              : static_cast<double>(jc / G - jc) * a.omega[pr];
            angle_cos_sin(ang0, c[e][hk], sn[e][hk]);
          }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
          for (int hk = 0; hk < 2; ++hk) {
            *reinterpret_cast<float4*>(cs + (8 * hk + kk) * CS_STRIDE + lane * 16) =
                make_float4(c[0][hk], c[1][hk], sn[0][hk], sn[1][hk]);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              float dc = fi_c[e], ds = fi_s[e];
              if (a.mode != 0) {
                const bool stay = ((j0 + 8 * hk + kk + 1) % G) == 0;
                dc = stay ? 1.f : pa_c[e];
                ds = stay ? 0.f : pa_s[e];
              }
              const float nc = c[e][hk] * dc - sn[e][hk] * ds;
              sn[e][hk] = sn[e][hk] * dc + c[e][hk] * ds;
              c[e][hk] = nc;
            }
          }
        }
      }
      mbar_arrive(&tbl[st]);  // every lane: its table entries are written
    }
    return;
  }
  if (warp >= nconsumers) return;  // fewer kv heads than warp pairs in this CTA

  // ---------------- consumers: warp pair (2h, 2h+1) handles kv head head0 + h ----------------
  const int hl = warp >> 1, nt = warp & 1;  // local kv head, n-tile (keys 8nt..8nt+7 of each stage)
  const int kvh = head0 + hl;
  const int g8 = lane >> 2, t4 = lane & 3;

  // query fragments (rows 0..g-1 = the g query heads of this kv head) under both RoPE forms,
  // fp16, in the m16n8k16 A layout: qa_*[kc] = {a0, a2} of k-chunk kc (rows 8..15 are zero)
  uint32_t qa_o[KC][2], qa_l[KC][2];
  bool q_fin = true;  // the rotated query fragments fit fp16
  {
    const bool row_ok = g8 < g;
    const __nv_bfloat16* qrow = a.q + (static_cast<long long>(bz) * a.hq + kvh * g + (row_ok ? g8 : 0)) * D;
    const double pl = (a.mode == 0) ? static_cast<double>(p) : static_cast<double>(p / G);
#pragma unroll
    for (int kc = 0; kc < KCP; ++kc)
#pragma unroll
      for (int sub = 0; sub < 2; ++sub) {
        const int d = 16 * kc + 8 * sub + 2 * t4;  // pair indices d, d + 1
        float xo[2], yo[2], xl[2], yl[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float x = 0.f, y = 0.f;
          if (row_ok) {
            x = __bfloat162float(qrow[d + e]);
            y = __bfloat162float(qrow[d + e + P]);
          }
          float c, sn;
          angle_cos_sin(static_cast<double>(p) * a.omega[d + e], c, sn);
          xo[e] = x * c - y * sn;
          yo[e] = y * c + x * sn;
          if (a.mode == 0)
            angle_cos_sin(pl * omega_long(d + e), c, sn);
          else
            angle_cos_sin(pl * a.omega[d + e], c, sn);
          xl[e] = x * c - y * sn;
          yl[e] = y * c + x * sn;
        }
        q_fin &= f16_ok(xo[0]) & f16_ok(xo[1]) & f16_ok(yo[0]) & f16_ok(yo[1]) & f16_ok(xl[0]) & f16_ok(xl[1]) &
                 f16_ok(yl[0]) & f16_ok(yl[1]);
        qa_o[kc][sub] = pack_f16x2(xo[0], xo[1]);
        qa_o[kc + KCP][sub] = pack_f16x2(yo[0], yo[1]);
        qa_l[kc][sub] = pack_f16x2(xl[0], xl[1]);
        qa_l[kc + KCP][sub] = pack_f16x2(yl[0], yl[1]);
      }
  }

  // O^T [D x 8 query rows]: o[mt][0..1] = d = 16mt + g8, rows 2t4, 2t4+1; o[mt][2..3] = d + 8
  float o[MT][4];
#pragma unroll
  for (int i = 0; i < MT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_r = -INFINITY, l_r = 0.f;  // softmax state of query row g8 (S layout)

  for (int s = 0; s < nstage; ++s) {
    const int st = s % NST;
    const int j0 = jbeg + s * KB;
    const int jt = j0 + nt * 8;  // first key of this warp's n-tile
    const bool tile_long = jt < local_from;
    const bool tile_local = jt + 7 >= local_from;
    // warp-uniform result: the ldmatrix / mma.sync below are warp-collective
    // the correction table is needed only when the stage holds long-range keys (its phase still
    // completes for every stage: the table warps arrive on each)
    if (!__all_sync(0xffffffffu, mbar_wait_abortable(&full[st], (s / NST) & 1, 2, &s_abort) &&
                                     (j0 >= local_from || mbar_wait_abortable(&tbl[st], (s / NST) & 1, 5, &s_abort)))) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      continue;
    }
    const uint8_t* cs = sCS + st * STAGE_CS;
    const uint32_t kbase = smem_u32(sK + st * STAGE_KV + hl * HALVES * HEAD_TILE);
    const uint32_t vbase = smem_u32(sV + st * STAGE_KV + hl * HALVES * HEAD_TILE);
    float so[4] = {0.f, 0.f, 0.f, 0.f}, sl[4] = {0.f, 0.f, 0.f, 0.f};
    const int krow = nt * 8 + (lane & 7);
    const int key_mine = nt * 8 + g8;  // key whose B elements this lane holds
#pragma unroll
    for (int kc = 0; kc < KCP; ++kc) {
      // lanes 0-7: d = 16kc.., 8-15: d + 8, 16-23: d + P, 24-31: d + 8 + P
      const int e_lo = 16 * kc + 8 * ((lane >> 3) & 1) + ((lane >> 4) ? P : 0);
      uint32_t r[4];
      ldmatrix_x4(r, kbase + (e_lo / 64) * HEAD_TILE + sw128(krow, (e_lo % 64) / 8));
      if (tile_local) {
        uint32_t a0[4] = {qa_o[kc][0], 0u, qa_o[kc][1], 0u};
        uint32_t a1[4] = {qa_o[kc + KCP][0], 0u, qa_o[kc + KCP][1], 0u};
        mma_f16_16816(so, a0, bf16x2_to_f16x2(r[0]), bf16x2_to_f16x2(r[1]));
        mma_f16_16816(so, a1, bf16x2_to_f16x2(r[2]), bf16x2_to_f16x2(r[3]));
      }
      if (tile_long) {
        // {cos d, cos d+1, sin d, sin d+1} of pairs d = 16kc + 2t4 (and d + 8), this lane's key
        const float4 c01 = *reinterpret_cast<const float4*>(cs + key_mine * CS_STRIDE + (16 * kc + 2 * t4) * 8);
        const float4 c89 = *reinterpret_cast<const float4*>(cs + key_mine * CS_STRIDE + (16 * kc + 8 + 2 * t4) * 8);
        // pair (x, y) -> (x c - y s, y c + x s), two pairs per packed fp32 instruction
        const uint32_t rx0 = rot_x(r[0], r[2], c01), ry0 = rot_y(r[0], r[2], c01);
        const uint32_t rx1 = rot_x(r[1], r[3], c89), ry1 = rot_y(r[1], r[3], c89);
        uint32_t a0[4] = {qa_l[kc][0], 0u, qa_l[kc][1], 0u};
        uint32_t a1[4] = {qa_l[kc + KCP][0], 0u, qa_l[kc + KCP][1], 0u};
        mma_f16_16816(sl, a0, rx0, rx1);
        mma_f16_16816(sl, a1, ry0, ry1);
      }
    }
    // merged scores of row g8 for keys jt + 2t4 + {0, 1}
    float sc[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int j = jt + 2 * t4 + e;
      float x = (j >= local_from) ? so[e] : sl[e];
      // An fp16 operand that overflowed (|x| >= 65520 rounds to inf) or a NaN key makes the
      // score inf or NaN (the padding query rows are zero: 0 * inf = NaN), so one test per
      // score covers every key operand of the stage.
      x *= a.scale_log2;
      if (j >= jend) x = -INFINITY;
      sc[e] = x;
    }
    // online softmax of row g8 over this n-tile
    float mx = fmaxf(sc[0], sc[1]);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_r, mx);
    const float ref = (m_new == -INFINITY) ? 0.f : m_new;
    const float alpha = fast_exp2(m_r - ref);
    m_r = m_new;
    const float p0 = fast_exp2(sc[0] - ref), p1 = fast_exp2(sc[1] - ref);
    l_r = l_r * alpha + (p0 + p1);
    // O^T columns are query rows 2t4 and 2t4 + 1: fetch their rescale factors
    const float al0 = __shfl_sync(0xffffffffu, alpha, 8 * t4);
    const float al1 = __shfl_sync(0xffffffffu, alpha, 8 * t4 + 4);
    // B = P^T: b0 = P[row g8][keys 2t4, 2t4 + 1] is exactly this lane's score pair
    const uint32_t pb = pack_bf16x2(p0, p1);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      o[mt][0] *= al0;
      o[mt][1] *= al1;
      o[mt][2] *= al0;
      o[mt][3] *= al1;
    }
    // Keys past the split's end (the last stage of a split, warp-uniform) have P = 0, but 0 * NaN
    // is NaN: their V rows hold whatever the cache (or a paged pool's slot) held, so this warp
    // zeroes its own rows of them before the PV products read them.
    const bool ragged = jt + 7 >= jend;
    if (ragged) {
      uint8_t* vrows = sV + st * STAGE_KV + hl * HALVES * HEAD_TILE;
#pragma unroll 1
      for (int r = 0; r < 8; ++r)
        if (jt + r >= jend && lane < 8)
#pragma unroll
          for (int hf = 0; hf < HALVES; ++hf)
            *reinterpret_cast<uint4*>(vrows + hf * HEAD_TILE + (nt * 8 + r) * 128 + lane * 16) = make_uint4(0, 0, 0, 0);
      __syncwarp();
    }
#pragma unroll
    for (int mt = 0; mt < MT; mt += 2) {
      // A = V^T: four 8x8 blocks (keys x d) of d-blocks 2mt .. 2mt+3, transposed by ldmatrix
      const int db = 2 * mt + (lane >> 3);
      uint32_t r[4];
      ldmatrix_x4_trans(r, vbase + (db / 8) * HEAD_TILE + sw128(krow, db % 8));
      mma_bf16_1688(o[mt], r[0], r[1], pb);
      mma_bf16_1688(o[mt + 1], r[2], r[3], pb);
    }
    // the zeroes above are generic-proxy writes to a slot the next TMA fill overwrites
    if (ragged) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }

  if (!q_fin) report_status(kDevRange, 42);
  // An fp16 key operand that overflowed (|x| >= 65520 rounds to inf) or a NaN key makes a score
  // inf or NaN (the padding query rows are zero: 0 * inf = NaN), which leaves the running max
  // at +inf or the running sum NaN: one test of the final state covers every key of the split.
  if (!(m_r < INFINITY) || !(l_r == l_r) || !(l_r < INFINITY)) report_status(kDevRange, 43);
  l_r += __shfl_xor_sync(0xffffffffu, l_r, 1);
  l_r += __shfl_xor_sync(0xffffffffu, l_r, 2);
  // The two warps of a kv head each hold the softmax state of their half of every stage; warp
  // nt = 1 hands its state to warp nt = 0 through shared memory (a named barrier per pair, 64
  // threads), which merges the two and writes one partial per split, halving what the combine
  // reads. Lane l of both warps holds the same rows and dimensions, so the merge is lane-wise.
  float* xo = reinterpret_cast<float*>(xch) + hl * (32 * (4 * MT + 2));
  if (nt == 1) {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) xo[(4 * mt + e) * 32 + lane] = o[mt][e];
    xo[(4 * MT) * 32 + lane] = m_r;
    xo[(4 * MT + 1) * 32 + lane] = l_r;
    asm volatile("bar.arrive %0, 64;" ::"r"(1 + hl) : "memory");
    return;
  }
  asm volatile("bar.sync %0, 64;" ::"r"(1 + hl) : "memory");
  {
    const float m1 = xo[(4 * MT) * 32 + lane], l1 = xo[(4 * MT + 1) * 32 + lane];
    const float M = fmaxf(m_r, m1);
    const float ref = (M == -INFINITY) ? 0.f : M;
    const float a0 = fast_exp2(m_r - ref), a1 = fast_exp2(m1 - ref);
    l_r = l_r * a0 + l1 * a1;
    m_r = M;
    // O^T columns are query rows 2t4 and 2t4 + 1: their factors sit on lanes 8t4 and 8t4 + 4
    const float f00 = __shfl_sync(0xffffffffu, a0, 8 * t4), f01 = __shfl_sync(0xffffffffu, a0, 8 * t4 + 4);
    const float f10 = __shfl_sync(0xffffffffu, a1, 8 * t4), f11 = __shfl_sync(0xffffffffu, a1, 8 * t4 + 4);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      o[mt][0] = o[mt][0] * f00 + xo[(4 * mt + 0) * 32 + lane] * f10;
      o[mt][1] = o[mt][1] * f01 + xo[(4 * mt + 1) * 32 + lane] * f11;
      o[mt][2] = o[mt][2] * f00 + xo[(4 * mt + 2) * 32 + lane] * f10;
      o[mt][3] = o[mt][3] * f01 + xo[(4 * mt + 3) * 32 + lane] * f11;
    }
  }
  // the merged partial of this split: rows < g
  const long long split = static_cast<long long>(bz) * a.parts_stride + blockIdx.x;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int row = 2 * t4 + e;
    if (row < g) {
      float* po = a.part_o + (split * a.hq + kvh * g + row) * D;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        po[16 * mt + g8] = o[mt][e];
        po[16 * mt + g8 + 8] = o[mt][2 + e];
      }
    }
  }
  if (t4 == 0 && g8 < g) {
    float* pml = a.part_ml + (split * a.hq + kvh * g + g8) * 2;
    pml[0] = m_r;
    pml[1] = l_r;
  }
}

template <int D>
constexpr int decode_smem_bytes() {
  return 2 * dec::NST * dec::HPC * (D / 64) * dec::KB * 128 + dec::NST * dec::KB * (D / 2 * 8 + 64) + 3 * dec::NST * 8 +
         dec::HPC * 32 * (4 * (D / 16) + 2) * 4;  // the warp pairs' exchange area
}

template <int D>
constexpr int decode_threads() {
  return (2 * dec::HPC + 3) * 32;  // consumers, TMA warp, two table warps
}

// Log-sum-exp merge of the split partials. CTA (h, dq) merges query head h for the 32
// dimensions 32dq .. 32dq+31, so D/32 CTAs share a head and the grid spreads over the SMs.
// The merge is latency-bound (it reads each partial once), so each warp issues the loads of NB
// of its splits at once and merges them online (running max, rescaled sum); one shared memory
// step then merges the warps. NB is the smallest of 2, 4, 8, 16 that covers a warp's share in
// one batch: a large NB costs registers (98 at NB = 16, two CTAs per SM), which a batched launch
// of many CTAs pays in waves, while a few CTAs over many splits want every load in flight.
constexpr int COMBINE_WARPS = 8;

// Batched (grid.z = sequence, seq_lens non-null): sequence b's partials start at row
// b * parts_stride, and only the ceil(seq_lens[b] / split_len) of its splits that hold keys
// were written; out / lse advance by hq rows per sequence.
template <int D, int NB>
__global__ void __launch_bounds__(32 * COMBINE_WARPS, NB <= 2 ? 8 : 1) decode_combine_kernel(
    const float* __restrict__ part_o, const float* __restrict__ part_ml, int n_split, int hq,
    __nv_bfloat16* __restrict__ out, float* __restrict__ lse, const int* __restrict__ seq_lens, int split_len,
    int parts_stride, int max_len) {
  __shared__ float red_acc[COMBINE_WARPS][32];
  __shared__ float red_l[COMBINE_WARPS];
  __shared__ float red_m[COMBINE_WARPS];
  pdl_wait();  // the partials of the previous kernel are complete and visible
  const int b = blockIdx.z;
  if (seq_lens) {
    const int Lb = seq_lens[b];
    // a length out of range had no partials written (the partial kernel reported it): merging
    // nothing gives 0 / 0, NaN, as this sequence's output
    n_split = (Lb >= 1 && Lb <= max_len) ? (Lb + split_len - 1) / split_len : 0;
    part_o += static_cast<long long>(b) * parts_stride * hq * D;
    part_ml += static_cast<long long>(b) * parts_stride * hq * 2;
    out += static_cast<long long>(b) * hq * D;
    if (lse) lse += static_cast<long long>(b) * hq;
  }
  const int h = blockIdx.x, d = 32 * blockIdx.y + (threadIdx.x & 31);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float m = -INFINITY, acc = 0.f, l = 0.f;  // this lane's running merge (log2 domain max)
  for (int s0 = warp; s0 < n_split; s0 += COMBINE_WARPS * NB) {
    float2 ml[NB];
    float ov[NB];
#pragma unroll
    for (int u = 0; u < NB; ++u) {
      const int sp = s0 + COMBINE_WARPS * u;
      ml[u] = make_float2(-INFINITY, 0.f);
      ov[u] = 0.f;
      if (sp < n_split) {
        const long long row = static_cast<long long>(sp) * hq + h;
        ml[u] = *reinterpret_cast<const float2*>(part_ml + row * 2);
        ov[u] = part_o[row * D + d];
      }
    }
#pragma unroll
    for (int u = 0; u < NB; ++u) {
      const float M = fmaxf(m, ml[u].x);
      const float ref = (M == -INFINITY) ? 0.f : M;
      const float c = fast_exp2(m - ref), w = fast_exp2(ml[u].x - ref);
      acc = acc * c + ov[u] * w;
      l = l * c + ml[u].y * w;
      m = M;
    }
  }
  red_acc[warp][lane] = acc;
  if (lane == 0) {
    red_l[warp] = l;
    red_m[warp] = m;
  }
  __syncthreads();
  if (warp == 0) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < COMBINE_WARPS; ++w) M = fmaxf(M, red_m[w]);
    const float ref = (M == -INFINITY) ? 0.f : M;
    float sa = 0.f, sl = 0.f;
#pragma unroll
    for (int w = 0; w < COMBINE_WARPS; ++w) {
      const float c = fast_exp2(red_m[w] - ref);
      sa += red_acc[w][lane] * c;
      sl += red_l[w] * c;
    }
    out[h * D + d] = __float2bfloat16(sa / sl);
    if (lse && blockIdx.y == 0 && lane == 0) lse[h] = (M + __log2f(sl)) * 0.69314718055994530942f;
  }
}

// Append: cache row p <- (R_orig(p) k_new, v_new). One warp per kv head.
struct AppendArgs {
  const __nv_bfloat16* k_new;  // [hkv, D]
  const __nv_bfloat16* v_new;  // [hkv, D]
  __nv_bfloat16* kcache;       // [cap, hkv, D]
  __nv_bfloat16* vcache;
  int hkv, p;
  double omega[64];
  // batched paged form (grid.y = sequence): position seq_lens[b] - 1, pool row via the block table
  const int* seq_lens;
  const int* block_table;
  int max_pages, page_size, pool_pages, max_len;
};

template <int D>
__global__ void decode_append_kernel(const __grid_constant__ AppendArgs a) {
  constexpr int P = D / 2;
  pdl_launch_dependents();  // the partial kernel may start; only its stage holding row p waits for us
  pdl_wait();               // launched early itself: the kernel before it (which may produce k_new) is done
  const int h = blockIdx.x, lane = threadIdx.x, b = blockIdx.y;
  const bool paged = a.seq_lens != nullptr;
  int p = a.p;  // logical position of the new token
  long long row = p;
  if (paged) {
    p = a.seq_lens[b] - 1;
    if (p < 0 || p >= a.max_len) {  // a length out of range: append nothing
      if (lane == 0) report_status(kDevIndex, 50);
      return;
    }
    const int pg = a.block_table[static_cast<long long>(b) * a.max_pages + p / a.page_size];
    if (pg < 0 || pg >= a.pool_pages) {  // a page outside the pool: write nothing
      if (lane == 0) report_status(kDevIndex, 51);
      return;
    }
    row = static_cast<long long>(pg) * a.page_size + p % a.page_size;
  }
  const __nv_bfloat16* kr = a.k_new + (static_cast<long long>(b) * a.hkv + h) * D;
  __nv_bfloat16* kd = a.kcache + (row * a.hkv + h) * D;
  for (int pr = lane; pr < P; pr += 32) {
    float c, s;
    angle_cos_sin(static_cast<double>(p) * a.omega[pr], c, s);
    const float x = __bfloat162float(kr[pr]), y = __bfloat162float(kr[pr + P]);
    kd[pr] = __float2bfloat16(x * c - y * s);
    kd[pr + P] = __float2bfloat16(y * c + x * s);
  }
  const __nv_bfloat16* vr = a.v_new + (static_cast<long long>(b) * a.hkv + h) * D;
  __nv_bfloat16* vd = a.vcache + (row * a.hkv + h) * D;
  for (int d = lane; d < D; d += 32) vd[d] = vr[d];
}

}  // namespace bf
