// Bifocal causal prefill, tcgen05 ping-pong form: two query tiles per CTA (D = 128).
//
// One CTA owns the same 128 query rows of two heads of one GQA group, so both tiles use
// every K and V tile it loads. Tensor memory (512 columns):
//   [  0, 128) S_A / P_A   [128, 256) S_B / P_B   [256, 384) O_A   [384, 512) O_B
// Q of both heads sits in shared memory (the A operand of QK^T), K/V tiles (128 keys)
// arrive by TMA into a ring of four 32 KB slots.
//
// Warp roles: warps 0..3 = softmax of tile A, warps 4..7 = softmax of tile B (a thread owns
// one query row; warp w reads TMEM lanes 32*(w%4)..), warp 8 = TMA producer, warp 9 = MMA
// issuer (one thread), warps 10..11 idle. Warps 8..11 form the third warpgroup only so that
// it can hand registers to the softmax warpgroups (setmaxnreg works per warpgroup): with 384
// threads the launch gives 168 registers per thread, the softmax rows need more than that to
// hold a 32-column S chunk and the whole row's P without spilling. The MMA thread issues,
// per visit v,
//   PV_A(v), QK_A(v+1), PV_B(v), QK_B(v+1)
// so while one tile's softmax runs, the tensor core works on the other tile: the two
// softmax groups never wait for each other.
//
// Visit order. Every key tile is scored with the branch that owns its pairs (ai-feeds
// summary of Jet-Long, 方法 key modules 1 and 3): the long-range RoPE forms when all pairs
// satisfy i - j >= w0, the original forms when all satisfy i - j < w0, and both (with
// complementary masks) when the band edge crosses the tile. The online softmax does not
// depend on the order of its terms, so the CTA takes all long-range visits first, then
// reloads Q with its original-RoPE form once, then takes the local visits. That keeps
// one Q form in shared memory at a time.
#pragma once
#include "common.cuh"
#include "prefill_tc.cuh"
#include "rope_loads.cuh"

namespace bf {
namespace tc2 {

using namespace tc;
constexpr int NSLOT2 = 4;
constexpr int NTHREADS2 = 384;  // 8 softmax warps, TMA warp, MMA warp, 2 idle warps (register donors)
constexpr uint32_t Q_BYTES = 32768;  // one Q tile, same layout as a K tile
constexpr uint32_t COL_SA = 0, COL_SB = 128, COL_OA = 256, COL_OB = 384;
constexpr int NK3 = 3, NV2 = 2;  // fused form: K ring and V ring
constexpr int kMaxSeqs = 64;     // sequences of one batched (paged) launch

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n"
      "}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]));
}

__device__ __forceinline__ int floordiv(int a, int b) { return a >= 0 ? a / b : -((-a + b - 1) / b); }

// Visit schedule of one query tile: n_lf fully long tiles (0..n_lf-1), then n_b band-edge
// tiles, then the rest fully local. Visits: long tiles, long half of band tiles, [Q reload],
// local half of band tiles (when w0 > 0), local tiles. The sliding-window kind drops the
// long-range pairs: its visits start after the `skip` long ones.
constexpr int KIND_PLAIN = 0, KIND_BIFOCAL = 1, KIND_WINDOW = 2;

struct Schedule {
  int n_kt, n_lf, n_b, n_bl, n_of, skip;
  __device__ __forceinline__ int n_long() const { return n_lf + n_b - skip; }
  __device__ __forceinline__ int total() const { return n_lf + n_b + n_bl + n_of - skip; }
  __device__ __forceinline__ void visit(int vis, int& t, int& kind) const {
    const int v = vis + skip;
    if (v < n_lf) {
      t = v;
      kind = LONG_FULL;
    } else if (v < n_lf + n_b) {
      t = v;  // band tiles follow the long tiles
      kind = LONG_ONLY;
    } else if (v < n_lf + n_b + n_bl) {
      t = n_lf + (v - n_lf - n_b);
      kind = ORIG_LOCAL;
    } else {
      t = n_lf + n_b + (v - n_lf - n_b - n_bl);
      kind = ORIG_FULL;
    }
  }
};

template <int KIND>
__device__ __forceinline__ Schedule make_schedule(int i0, int n_kt, int w0) {
  Schedule s;
  s.n_kt = n_kt;
  s.skip = 0;
  if (KIND == KIND_PLAIN) {
    s.n_lf = s.n_b = s.n_bl = 0;
    s.n_of = n_kt;
    return s;
  }
  const int A = floordiv(i0 - (BN - 1) - w0, BN);      // tiles t <= A: every pair long-range
  const int C = floordiv(i0 + (BM - 1) - w0, BN) + 1;  // tiles t >= C: every pair local
  s.n_lf = min(max(A + 1, 0), n_kt);
  s.n_b = max(min(C, n_kt) - s.n_lf, 0);
  s.n_bl = w0 > 0 ? s.n_b : 0;
  s.n_of = n_kt - s.n_lf - s.n_b;
  if (KIND == KIND_WINDOW) s.skip = s.n_lf + s.n_b;
  return s;
}

}  // namespace tc2

struct Tc2Args {
  // FUSED = false: the RoPE pass's fp16 operand forms, [b*h][L][128], box (64, 128, 1).
  // FUSED = true: qo_map is the raw bf16 q [b][Lq][hq][128] and ko_map the raw bf16 keys
  // [b][L][hkv][128] (or the cache of original-RoPE keys), box (64, 1, 128, 1); ql/kl unused.
  CUtensorMap qo_map;
  CUtensorMap ql_map;
  CUtensorMap ko_map;
  CUtensorMap kl_map;
  CUtensorMap v_map;   // bf16 [b][L][hkv][128], box (64, 1, 128, 1)
  __nv_bfloat16* out;  // [b, Lq, hq, 128]
  float* lse;          // [b, hq, Lq] or null
  int L, hq, hkv, batch, w0;
  // query rows: Lq rows at absolute positions q_off .. q_off + Lq - 1 (a full prefill has
  // q_off = 0 and Lq = L; a chunk over a cache has q_off = the cached length); keys 0 .. L-1
  int q_off, Lq;
  float scale_log2;
  RopeSrc src;  // angles of the fused loads (FUSED only)
  int test_skip_fill;  // test only (bifocal_test_set_fault): 1 + the fill CTA 0's producer never issues; 0 = off
  // A batch of chunks over a paged cache (FUSED only, nseq > 0). Launch-order entry s is the
  // chunk of sequence seq_id[s] (its block-table row): cached length seq_P0[s], chunk length
  // seq_C[s], factor seq_G[s], first row seq_qrow[s] of the packed q / out / lse rows (total_rows
  // in all); query tiles tile_start[s] .. tile_start[s + 1] - 1 of the grid are its. Key j of
  // that sequence is pool row block_table[seq_id[s] * max_pages + j / page_size] * page_size +
  // j % page_size, and K / V tiles arrive in segments of seg_rows = min(page_size, 128) rows.
  int nseq, total_rows;
  const int* block_table;
  int max_pages, page_size, seg_rows;
  int pool_pages;  // a block-table entry outside [0, pool_pages) is reported and its segment read as zeros
  int tile_start[tc2::kMaxSeqs + 1];
  int seq_id[tc2::kMaxSeqs], seq_P0[tc2::kMaxSeqs], seq_C[tc2::kMaxSeqs], seq_G[tc2::kMaxSeqs],
      seq_qrow[tc2::kMaxSeqs];
};

// FUSED = false: Q and K tiles come by TMA from the RoPE pass's fp16 forms; K and V share a
// ring of four slots (fill n in slot n % 4: K of visit v is fill 2v, V fill 2v + 1).
// FUSED = true: TMA brings the raw bf16 tiles; warps 10 and 11 rotate Q and K in place into
// fp16 operands (rope_loads.cuh); K has its own ring of three slots, V of two. No rotated
// copy of q or k exists in HBM.
template <int KIND, bool FUSED>
__global__ void __launch_bounds__(tc2::NTHREADS2, 1) attn_tc2_kernel(const __grid_constant__ Tc2Args a) {
  using namespace tc2;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ uint64_t full[NSLOT2], empty[NSLOT2], s_full[2], p_ready[2], o_done[2], q_full, q_free, mma_drain;
  // P is handed over in two halves (keys 0-63, 64-127 of the tile): p_lo releases the first
  // half's P.V while the softmax finishes the second; o_lo completes when that half's P.V has
  // run (waited on only when the second half needs a new row reference after the first was sent)
  __shared__ uint64_t p_lo[2], o_lo[2];
  // fused rings: K raw landed / K operand ready / K slot free; V landed / V slot free; raw Q landed
  __shared__ uint64_t kraw[NK3], kfull[NK3], kempty[NK3], vfull[NV2], vempty[NV2], q_raw, v_fix[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pairs = a.hq / 2;
  // This CTA's query tile: rows q_off + qt*BM .. of a sequence with Lq query rows after q_off
  // cached ones (L = q_off + Lq keys), factor G; b is its batch index (dense) or block-table
  // row (paged); qrow0 its first row in out / lse.
  int qt, hp, b, q_off, Lq, L, G, qrow0;
  const bool paged = FUSED && a.nseq > 0;
  if (paged) {
    const int tile = static_cast<int>(blockIdx.x) / pairs;
    hp = static_cast<int>(blockIdx.x) % pairs;
    int sq = 0;
    while (sq + 1 < a.nseq && a.tile_start[sq + 1] <= tile) ++sq;
    b = a.seq_id[sq];
    q_off = a.seq_P0[sq];
    Lq = a.seq_C[sq];
    G = a.seq_G[sq];
    qrow0 = a.seq_qrow[sq];
    qt = (Lq + BM - 1) / BM - 1 - (tile - a.tile_start[sq]);  // heaviest first within the sequence
  } else {
    // kv-head major: the CTAs resident at one time share one kv head's K and V tiles (the key
    // forms of one head fit in L2 at 128K, those of all eight do not: with the query tiles of
    // every head in flight, K and V were read from DRAM ~23 times over), heaviest query tile
    // first within a head
    const int n_qt = (a.Lq + BM - 1) / BM;
    const int ppk = pairs / a.hkv;  // head pairs per kv head
    const int idx = static_cast<int>(blockIdx.x);
    const int pk = idx % ppk;
    const int rest = idx / ppk;
    qt = n_qt - 1 - rest % n_qt;
    const int bk = rest / n_qt;  // batch * hkv + kv head
    b = bk / a.hkv;
    hp = (bk % a.hkv) * ppk + pk;
    q_off = a.q_off;
    Lq = a.Lq;
    G = a.src.G;
    qrow0 = b * a.Lq;
  }
  L = q_off + Lq;
  const int h0 = 2 * hp;  // heads h0 (tile A) and h0 + 1 (tile B), same kv head
  const int kvh = h0 / (a.hq / a.hkv);
  const int i0 = q_off + qt * BM;  // absolute position of the tile's first query row
  const int n_kt = (min(i0 + BM, L) + BN - 1) / BN;
  const Schedule sch = make_schedule<KIND>(i0, n_kt, a.w0);
  const int nv = sch.total();
  const bool has_long = sch.n_long() > 0;
  const bool has_orig = sch.n_bl + sch.n_of > 0;
  const bool reload_q = has_long && has_orig;
  const int v_sw = sch.n_long();  // first local visit (when reload_q)
  const uint32_t qbase = smem_u32(smem);                  // Q_A, Q_B
  const uint32_t slots = qbase + 2 * Q_BYTES;             // K/V ring; fused: K slots, then V slots
  const uint32_t vslots = slots + (FUSED ? NK3 : 0) * SLOT_BYTES;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int i = 0; i < NSLOT2; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < NK3; ++i) {
      mbar_init(&kraw[i], 1);
      mbar_init(&kfull[i], rl::NXF);
      mbar_init(&kempty[i], 1);
    }
    for (int i = 0; i < NV2; ++i) {
      mbar_init(&vfull[i], 1);
      mbar_init(&vempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_ready[i], 4);
      mbar_init(&p_lo[i], 4);
      mbar_init(&o_done[i], 1);
      mbar_init(&o_lo[i], 1);
    }
    mbar_init(&q_raw, 1);
    mbar_init(&v_fix[0], rl::NXF);  // one per visit of a tile past a paged sequence's end (at most two:
    mbar_init(&v_fix[1], rl::NXF);  // its long-range half and its local half), each used once
    mbar_init(&q_full, FUSED ? rl::NXF : 1);
    mbar_init(&q_free, 1);
    mbar_init(&mma_drain, 1);
    fence_barrier_init();
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                 "r"(NCOLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = tmem_base_sh;

  // Barriers and slots of visit v's K and V tiles, for either ring layout.
  auto k_full = [&](int v) -> uint64_t* { return FUSED ? &kfull[v % NK3] : &full[(2 * v) % NSLOT2]; };
  auto k_full_ph = [&](int v) -> uint32_t { return FUSED ? (v / NK3) & 1 : ((2 * v) / NSLOT2) & 1; };
  auto k_empty = [&](int v) -> uint64_t* { return FUSED ? &kempty[v % NK3] : &empty[(2 * v) % NSLOT2]; };
  auto k_slot = [&](int v) -> int { return FUSED ? v % NK3 : (2 * v) % NSLOT2; };
  auto v_full = [&](int v) -> uint64_t* { return FUSED ? &vfull[v % NV2] : &full[(2 * v + 1) % NSLOT2]; };
  auto v_full_ph = [&](int v) -> uint32_t { return FUSED ? (v / NV2) & 1 : ((2 * v + 1) / NSLOT2) & 1; };
  auto v_empty = [&](int v) -> uint64_t* { return FUSED ? &vempty[v % NV2] : &empty[(2 * v + 1) % NSLOT2]; };
  auto v_slot = [&](int v) -> int { return FUSED ? v % NV2 : (2 * v + 1) % NSLOT2; };

  // Registers: launched at 168 per thread (384 threads). Warpgroup 2 (TMA, MMA, two idle or
  // transform warps) gives 72 of them back and the two softmax warpgroups take 32 more each:
  // 2 * 128 * 200 + 128 * 96 = 63488 <= 384 * 168, so the increase never waits for registers
  // that the block does not hold. Each role branch starts with its own setmaxnreg so that the
  // compiler allocates each branch within its own limit.
  if (warp >= 8) {
    // the fused form's transform warps take the 8 registers left over: 2 * 128 * 200 + 128 * 104
    // = 384 * 168 exactly
    if (FUSED)
      asm volatile("setmaxnreg.dec.sync.aligned.u32 104;");
    else
      asm volatile("setmaxnreg.dec.sync.aligned.u32 96;");
    if (warp == 8) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        prefetch_tensormap(&a.qo_map);
        prefetch_tensormap(&a.ko_map);
        prefetch_tensormap(&a.v_map);
        if (KIND == KIND_BIFOCAL && !FUSED) {
          prefetch_tensormap(&a.ql_map);
          prefetch_tensormap(&a.kl_map);
        }
        const int skip = blockIdx.x == 0 ? a.test_skip_fill - 1 : -1;  // test only: never issue this fill
        uint32_t used = 0, par = 0;    // unfused ring: per slot, has a fill been issued, parity of the fills
        uint32_t kused = 0, kpar = 0;  // fused K ring (raw landed barriers)
        uint32_t vused = 0, vpar = 0;  // fused V ring
        // Q: both heads; fused: raw rows of this call (map over Lq rows), else the rotated form
        auto load_q = [&](bool lng) {
          uint64_t* bar = FUSED ? &q_raw : &q_full;
          mbar_arrive_expect_tx(bar, 2 * Q_BYTES);
          for (int x = 0; x < 2; ++x) {
            uint8_t* dst = smem + x * Q_BYTES;
            if (FUSED) {
              // raw rows [b][Lq][hq][128], or the packed rows of a paged batch [1][total_rows][hq][128]
              const int row = (paged ? qrow0 : 0) + qt * BM, bb = paged ? 0 : b;
              tma_load_4d(dst, &a.qo_map, bar, 0, h0 + x, row, bb);
              tma_load_4d(dst + HALF_BYTES, &a.qo_map, bar, 64, h0 + x, row, bb);
            } else {
              const CUtensorMap* m = lng ? &a.ql_map : &a.qo_map;
              tma_load_3d(dst, m, bar, 0, qt * BM, b * a.hq + h0 + x);
              tma_load_3d(dst + HALF_BYTES, m, bar, 64, qt * BM, b * a.hq + h0 + x);
            }
          }
        };
        load_q(has_long);
        int q_loads = 1;
        const int krow = b * a.hkv + kvh;
        // One fill: the K (x = 0) or V (x = 1) tile of visit v, fill number 2v + x, into its slot
        // once the slot's previous tile is consumed. False when a wait gave up.
        auto fill = [&](int x, int v) -> bool {
          const int n = 2 * v + x;
          const int use = FUSED ? (x == 0 ? v / NK3 : v / NV2) : n / NSLOT2;
          uint64_t* freed = x == 0 ? k_empty(v) : v_empty(v);
          if (use > 0 && !mbar_wait_abortable(freed, (use - 1) & 1, 10, &s_abort)) return false;
          if (n == skip) return true;
          int t, kind;
          sch.visit(v, t, kind);
          const bool lng = kind == LONG_FULL || kind == LONG_ONLY;
          const int sl = x == 0 ? k_slot(v) : v_slot(v);
          if (FUSED) {
            if (x == 0) {
              kused |= 1u << sl;
              kpar ^= 1u << sl;
            } else {
              vused |= 1u << sl;
              vpar ^= 1u << sl;
            }
          } else {
            used |= 1u << sl;
            par ^= 1u << sl;
          }
          uint64_t* bar = FUSED ? (x == 0 ? &kraw[sl] : &vfull[sl]) : &full[sl];
          uint8_t* dst = smem + ((x == 0 ? slots : vslots) - qbase) + sl * SLOT_BYTES;
          if (paged) {
            // segments of seg_rows keys, each one page's rows of the pool; segments wholly past
            // the sequence's end are not loaded (their K rows are zeroed by the transform, their
            // V rows by the fix-up of each visit of that tile)
            const CUtensorMap* m = x == 0 ? &a.ko_map : &a.v_map;
            const int nseg = BN / a.seg_rows;
            const int nvalid = min(nseg, (L - t * BN + a.seg_rows - 1) / a.seg_rows);
            mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nvalid * a.seg_rows) * 256u);
            for (int sg = 0; sg < nvalid; ++sg) {
              const int j = t * BN + sg * a.seg_rows;
              const int pg = a.block_table[static_cast<long long>(b) * a.max_pages + j / a.page_size];
              const bool pg_ok = pg >= 0 && pg < a.pool_pages;
              if (!pg_ok) report_status(kDevIndex, 55);
              // a bad entry loads the box that starts just past the pool's last row: TMA fills it with zeros
              const int row = pg_ok ? pg * a.page_size + j % a.page_size : a.pool_pages * a.page_size;
              uint8_t* d0 = dst + sg * a.seg_rows * 128;
              tma_load_4d(d0, m, bar, 0, kvh, row, 0);
              tma_load_4d(d0 + HALF_BYTES, m, bar, 64, kvh, row, 0);
            }
            return true;
          }
          mbar_arrive_expect_tx(bar, SLOT_BYTES);
          if (x == 1 || FUSED) {
            const CUtensorMap* m = x == 0 ? &a.ko_map : &a.v_map;
            tma_load_4d(dst, m, bar, 0, kvh, t * BN, b);
            tma_load_4d(dst + HALF_BYTES, m, bar, 64, kvh, t * BN, b);
          } else {
            const CUtensorMap* m = lng ? &a.kl_map : &a.ko_map;
            tma_load_3d(dst, m, bar, 0, t * BN, krow);
            tma_load_3d(dst + HALF_BYTES, m, bar, 64, t * BN, krow);
          }
          return true;
        };
        if (FUSED) {
          // K runs two visits ahead of V (step u: K(u), then V(u - 2)), so no K fill waits behind
          // a V slot: a raw K tile still has to be rotated after it lands. The raw Q reload goes
          // out as soon as q_free has completed: tried at step v_sw, waited for at step v_sw + 1,
          // after V(v_sw - 1), the last fill the MMA needs before it can reach q_free.
          bool q_pending = reload_q;
          for (int u = 0; u < nv + 2; ++u) {
            if (u < nv && !fill(0, u)) break;
            if (u >= 2 && u - 2 < nv && !fill(1, u - 2)) break;
            if (q_pending && u >= v_sw) {
              if (u > v_sw || mbar_try_wait(&q_free, 0)) {
                if (!mbar_wait_abortable(&q_free, 0, 12, &s_abort)) break;
                load_q(false);
                ++q_loads;
                q_pending = false;
              }
            }
          }
        } else {
          for (int v = 0; v < nv; ++v) {
            if (reload_q && v == v_sw) {
              // every QK^T with the long-range Q has finished reading it
              if (!mbar_wait_abortable(&q_free, 0, 12, &s_abort)) break;
              load_q(false);
              ++q_loads;
            }
            if (!fill(0, v) || !fill(1, v)) break;
          }
        }
        // drain: every copy issued must have landed before the CTA may exit: the last fill of
        // every slot (the ones before it were consumed, or a later fill could not have been
        // issued) and the last Q load; the waits sleep between polls, so they take no issue
        // slots from the warps still working
        if (FUSED) {
          for (int sl = 0; sl < NK3; ++sl)
            if (kused & (1u << sl)) mbar_wait_sleepy(&kraw[sl], ((kpar >> sl) & 1u) ^ 1u, 11);
          for (int sl = 0; sl < NV2; ++sl)
            if (vused & (1u << sl)) mbar_wait_sleepy(&vfull[sl], ((vpar >> sl) & 1u) ^ 1u, 11);
          mbar_wait_sleepy(&q_raw, (q_loads - 1) & 1, 13);
        } else {
          for (int sl = 0; sl < NSLOT2; ++sl)
            if (used & (1u << sl)) mbar_wait_sleepy(&full[sl], ((par >> sl) & 1u) ^ 1u, 11);
          mbar_wait_sleepy(&q_full, (q_loads - 1) & 1, 13);
        }
      }
    } else if (FUSED && warp >= 10) {
      // ------------------------------------------------------------ fused RoPE: rotate tiles in place
      const int pt = (warp - 10) * 32 + lane;
      const int cch = pt & 7, r0 = pt >> 3;
      // Q: raw rows landed -> the first form (long-range when the tile has long visits)
      if (warp_wait(&q_raw, 0, 14, &s_abort)) {
        rope_query_tiles(qbase, a.src, G, has_long ? rl::FORM_LONG : rl::FORM_ORIG, i0, cch, r0);
        fence_proxy_async_smem();
        mbar_arrive(&q_full);
        Rot8 st, s8;
        int cur_form = -1, next_t = -1, run = 0;
        int n_fixed = 0;  // visits of a tile past a paged sequence's end handled so far
        for (int v = 0; v < nv; ++v) {
          int t, kind;
          sch.visit(v, t, kind);
          const int form = (kind == LONG_FULL || kind == LONG_ONLY) ? rl::FORM_LONG : rl::FORM_ORIG;
          const int sl = v % NK3;
          if (!warp_wait(&kraw[sl], (v / NK3) & 1, 16, &s_abort)) break;
          const bool linear = form_linear(a.src, G, form);
          if (linear && !(a.src.cache && form == rl::FORM_ORIG)) {
            if (form != cur_form) rot_step(s8, a.src, G, form, true, 8, 8 * cch);
            if (form != cur_form || t != next_t || run >= rl::ANCHOR_EVERY) {
              rot_exact(st, a.src, G, form, true, static_cast<long long>(t) * BN + r0, 8 * cch);
              run = 0;
            }
            cur_form = form;
            next_t = t + 1;
            ++run;
          } else {
            cur_form = -1;  // st is not kept (exact angles per row, or no rotation): anchor the next run
          }
          rope_key_tile(slots + sl * SLOT_BYTES, a.src, G, form, linear, t * BN, L, cch, r0, st, s8);
          fence_proxy_async_smem();
          mbar_arrive(&kfull[sl]);
          if (paged && t * BN + BN > L && n_fixed < 2) {
            // this tile runs past the sequence's end (it may be visited twice, once per branch):
            // its V rows there hold whatever the pool holds; zero them once the tile has landed
            // (the MMA waits for v_fix before this visit's PV)
            if (!warp_wait(&vfull[v % NV2], (v / NV2) & 1, 18, &s_abort)) break;
            zero_tile_rows(vslots + (v % NV2) * SLOT_BYTES, L - t * BN, cch, r0);
            fence_proxy_async_smem();
            mbar_arrive(&v_fix[n_fixed++]);
          }
          if (reload_q && v == v_sw) {
            // the first original-form visit's K is ready; now the original-form Q: the producer
            // reloads the raw rows once every long-range QK^T has read the first form
            if (!warp_wait(&q_raw, 1, 15, &s_abort)) break;
            rope_query_tiles(qbase, a.src, G, rl::FORM_ORIG, i0, cch, r0);
            fence_proxy_async_smem();
            mbar_arrive(&q_full);
          }
        }
      }
    } else if (warp == 9) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0 && nv > 0) {
        int n_fix = 0;  // visits of a tile past the sequence's end seen so far (paged: V tail zeroed)
        bool ok = mbar_wait_abortable(&q_full, 0, 20, &s_abort);
        fence_after();
        // The issuing thread waits on each tcgen05.mma before it can issue the next one, so any
        // arithmetic between two MMAs of a group adds to the group's time (it halved the tensor
        // rate here). Descriptors are therefore formed once, and the eight K-steps of a group
        // only add constants to the start-address field (addresses stay below 2^18, so the
        // field never carries into the next one).
        const uint64_t dqa = k_desc(qbase, 0), dqb = k_desc(qbase + Q_BYTES, 0);
        const uint64_t dk0 = k_desc(slots, 0), dv0 = v_desc(vslots, 0);
        auto qk = [&](int x, int v) {
          const uint64_t a0 = x == 0 ? dqa : dqb;
          const uint64_t b0 = dk0 + static_cast<uint64_t>(k_slot(v) * (SLOT_BYTES >> 4));
          const uint32_t d = tmem + (x == 0 ? COL_SA : COL_SB);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t step = ((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4;
            mma_ss(d, a0 + step, b0 + step, IDESC_QK, kk > 0);
          }
          mma_commit(&s_full[x]);
        };
        // O_x += P_x(v) V(v) over keys 64h .. 64h + 63 (four 16-key steps); h = 0 commits o_lo, h = 1 o_done
        auto pv_half = [&](int x, int v, int h) {
          const uint64_t b0 = dv0 + static_cast<uint64_t>(v_slot(v) * (SLOT_BYTES >> 4));
          const uint32_t p_col = tmem + (x == 0 ? COL_SA : COL_SB);
          const uint32_t o_col = tmem + (x == 0 ? COL_OA : COL_OB);
          const uint32_t acc0 = v > 0;
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const int kk = 4 * h + k4;
            mma_ts(o_col, p_col + kk * 8, b0 + static_cast<uint64_t>(kk * (2048 >> 4)), IDESC_PV, kk > 0 ? 1u : acc0);
          }
          mma_commit(h == 0 ? &o_lo[x] : &o_done[x]);
        };
        // visit 0: S_A, S_B
        if (ok) ok = mbar_wait_abortable(k_full(0), k_full_ph(0), 21, &s_abort);
        if (ok) {
          fence_after();
          qk(0, 0);
          qk(1, 0);
          mma_commit(k_empty(0));
          if (reload_q && v_sw == 1) mma_commit(&q_free);
        }
        for (int v = 0; v < nv && ok; ++v) {
          // O_A += P_A(v) V(v), first half as soon as the softmax has sent it
          if (!mbar_wait_abortable(&p_lo[0], v & 1, 22, &s_abort) ||
              !mbar_wait_abortable(v_full(v), v_full_ph(v), 23, &s_abort)) {
            ok = false;
            break;
          }
          if (paged) {
            int tv, kv;
            sch.visit(v, tv, kv);
            if (tv * BN + BN > L && n_fix < 2 && !mbar_wait_abortable(&v_fix[n_fix++], 0, 28, &s_abort)) {
              ok = false;
              break;
            }
          }
          fence_after();
          pv_half(0, v, 0);
          if (!mbar_wait_abortable(&p_ready[0], v & 1, 29, &s_abort)) {
            ok = false;
            break;
          }
          fence_after();
          pv_half(0, v, 1);
          const bool more = v + 1 < nv;
          if (more) {
            if (reload_q && v + 1 == v_sw && !mbar_wait_abortable(&q_full, 1, 24, &s_abort)) {
              ok = false;
              break;
            }
            if (!mbar_wait_abortable(k_full(v + 1), k_full_ph(v + 1), 25, &s_abort)) {
              ok = false;
              break;
            }
            fence_after();
            qk(0, v + 1);  // S_A is free: PV_A(v) was issued before
          }
          // O_B += P_B(v) V(v)
          if (!mbar_wait_abortable(&p_lo[1], v & 1, 26, &s_abort)) {
            ok = false;
            break;
          }
          fence_after();
          pv_half(1, v, 0);
          if (!mbar_wait_abortable(&p_ready[1], v & 1, 33, &s_abort)) {
            ok = false;
            break;
          }
          fence_after();
          pv_half(1, v, 1);
          mma_commit(v_empty(v));
          if (more) {
            qk(1, v + 1);
            mma_commit(k_empty(v + 1));
            if (reload_q && v + 2 == v_sw) mma_commit(&q_free);
          }
        }
        // every MMA issued has finished before teardown
        mma_commit(&mma_drain);
        mbar_wait(&mma_drain, 0, 27);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 200;");
    // ------------------------------------------------------------ softmax warps: 0..3 tile A, 4..7 tile B
    const int x = warp >> 2;        // tile
    const int quad = warp & 3;      // TMEM lane quadrant this warp may access
    const int r = quad * 32 + lane;
    const int i = i0 + r;
    const int h = h0 + x;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t s_col = lane_addr + (x == 0 ? COL_SA : COL_SB);
    const uint32_t o_col = lane_addr + (x == 0 ? COL_OA : COL_OB);
    const float sc = a.scale_log2;
    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = true;
    for (int v = 0; v < nv && ok; ++v) {
      int t, kind;
      sch.visit(v, t, kind);
      const int j0 = t * BN;
      // every lane waits; the result is made warp-uniform because the TMEM accesses below
      // are warp-collective (.sync.aligned)
      if (!__all_sync(0xffffffffu, mbar_wait_abortable(&s_full[x], v & 1, 30, &s_abort))) {
        ok = false;
        break;
      }
      fence_after();
      const bool masked = kind != LONG_FULL && (kind != ORIG_FULL || j0 + BN - 1 > i0);
      const int lo = (kind == LONG_ONLY) ? a.w0 : 0;            // keep lo <= i - j
      const int hi = (kind == ORIG_LOCAL) ? a.w0 : 0x7fffffff;  //      and i - j < hi
      float alpha = 1.f, rs = 0.f;
      bool grow = false;
      uint32_t pk[64];  // P of the whole row, bf16 pairs (keys 2u, 2u + 1 in pk[u])
      // Fast path (unmasked visits once the row has a reference): one pass with the current
      // reference m_ref, half a row at a time. m_ref never exceeds the running max, so every P
      // term is bounded by 2^(running max - m_ref); a half whose sum stays within 2^24 has no
      // term that could overflow. The first half (keys 0-63) goes to the MMA as soon as it is
      // known to be safe, so its P.V runs while the second half is computed. A first half above
      // 2^24 (or not finite) sends the visit to the exact two-pass path below; a second half
      // above it, after the first was sent, takes a new reference for the second half and
      // rescales O once the first half's P.V has run (o_lo).
      // Every choice is made for the whole warp: each path reads S with tcgen05.ld, a
      // warp-collective (.sync.aligned) instruction, so the lanes must not split between them.
      // A row that needs the exact path (its reference is still -inf: no key of the earlier
      // visits was in range, as happens in a sliding window; or its fast sum overflowed) takes
      // the whole warp with it; the exact path is correct for every row.
      bool exact = __any_sync(0xffffffffu, masked || m_ref == -INFINITY);
      bool lo_sent = false;
      if (!exact) {
        // pairs of columns go through the packed f32x2 FMA and add
        const uint64_t sc2 = f2_pack(sc, sc);
        auto half_pass = [&](int c_lo, uint64_t nref2) -> float {
          uint64_t r4[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) r4[u] = f2_pack(0.f, 0.f);
#pragma unroll
          for (int c0 = c_lo; c0 < c_lo + 64; c0 += 32) {
            float s[32];
            tmem_ld32(s_col + c0, s);
            wait_ld();
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              float x0, x1;
              f2_unpack(f2_fma(f2_pack(s[c], s[c + 1]), sc2, nref2), x0, x1);
              const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
              r4[(c >> 1) & 3] = f2_add(r4[(c >> 1) & 3], f2_pack(p0, p1));
              pk[(c0 + c) >> 1] = pack_bf16x2(p0, p1);
            }
          }
          float r8[8];
#pragma unroll
          for (int u = 0; u < 4; ++u) f2_unpack(r4[u], r8[2 * u], r8[2 * u + 1]);
          return ((r8[0] + r8[1]) + (r8[2] + r8[3])) + ((r8[4] + r8[5]) + (r8[6] + r8[7]));
        };
        const float rs_lo = half_pass(0, f2_pack(-m_ref, -m_ref));
        exact = __any_sync(0xffffffffu, !(rs_lo <= 16777216.f));
        if (!exact) {
          // send the first half: P over columns 0-31 of the S buffer (S of keys 0-63 is consumed)
          tmem_st32(s_col, pk);
          wait_st();
          fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_lo[x]);
          lo_sent = true;
          float rs_hi = half_pass(64, f2_pack(-m_ref, -m_ref));
          rs = rs_lo + rs_hi;
          if (__any_sync(0xffffffffu, !(rs_hi <= 16777216.f))) {
            // Rare: the second half's terms outgrow the reference the first half was sent with.
            // Its S columns (64-127) are intact: take the raw max over them, move the reference
            // where it grew past the threshold, and recompute the second half against it.
            float m8[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) m8[u] = -INFINITY;
#pragma unroll
            for (int c0 = 64; c0 < 128; c0 += 32) {
              float s[32];
              tmem_ld32(s_col + c0, s);
              wait_ld();
#pragma unroll
              for (int c = 0; c < 32; c += 8)
#pragma unroll
                for (int u = 0; u < 8; ++u) m8[u] = fmaxf(m8[u], s[c + u]);
            }
            const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                   fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) *
                             sc;
            if (mx > m_ref + RESCALE_THRESHOLD) {
              alpha = fast_exp2(m_ref - mx);
              grow = true;
              m_ref = mx;
            }
            rs_hi = half_pass(64, f2_pack(-m_ref, -m_ref));
            rs = rs_lo * alpha + rs_hi;  // l_sum * alpha + rs below: both earlier sums rescaled
            // O must hold the first half's P.V (old reference) before it is rescaled, and the
            // second half's P.V (new reference) must not start before: it waits for p_ready
            if (!__all_sync(0xffffffffu, mbar_wait_abortable(&o_lo[x], v & 1, 34, &s_abort))) {
              ok = false;
              break;
            }
            fence_after();
            if (__any_sync(0xffffffffu, grow)) {  // warp-uniform; rows that need none scale by 1
              const float f = grow ? alpha : 1.f;
#pragma unroll 1
              for (int c0 = 0; c0 < 128; c0 += 32) {
                float ov[32];
                tmem_ld32(o_col + c0, ov);
                wait_ld();
                uint32_t ou[32];
#pragma unroll
                for (int u = 0; u < 32; ++u) ou[u] = __float_as_uint(ov[u] * f);
                tmem_st32(o_col + c0, ou);
              }
            }
          }
          l_sum = l_sum * alpha + rs;
          tmem_st32(s_col + 32, pk + 32);  // the second half: columns 32-63
        }
      }
      if (exact) {
        // pass 1: raw row max over the 128 columns
        float m8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) m8[u] = -INFINITY;
#pragma unroll
        for (int c0 = 0; c0 < 128; c0 += 32) {
          float s[32];
          tmem_ld32(s_col + c0, s);
          wait_ld();
          if (masked) {
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const int d = i - (j0 + c0 + c);
              s[c] = (d >= lo && d < hi) ? s[c] : -INFINITY;
            }
          }
#pragma unroll
          for (int c = 0; c < 32; c += 8)
#pragma unroll
            for (int u = 0; u < 8; ++u) m8[u] = fmaxf(m8[u], s[c + u]);
        }
        const float mx =
            fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) *
            sc;
        // lazy rescale: a row keeps its reference unless its max grew by more than the threshold
        if (mx > m_ref + RESCALE_THRESHOLD || (m_ref == -INFINITY && mx > -INFINITY)) {
          alpha = (m_ref == -INFINITY) ? 0.f : fast_exp2(m_ref - mx);
          grow = m_ref != -INFINITY;  // O already holds this row's earlier terms
          m_ref = mx;
        }
        const float neg_ref = (m_ref == -INFINITY) ? 0.f : -m_ref;
        // pass 2: P = exp2(s * scale - ref)
        float r8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c0 = 0; c0 < 128; c0 += 32) {
          float s[32];
          tmem_ld32(s_col + c0, s);
          wait_ld();
          if (masked) {
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const int d = i - (j0 + c0 + c);
              s[c] = (d >= lo && d < hi) ? s[c] : -INFINITY;
            }
          }
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float p0 = fast_exp2(fmaf(s[c], sc, neg_ref)), p1 = fast_exp2(fmaf(s[c + 1], sc, neg_ref));
            r8[(c >> 1) & 7] += p0 + p1;
            pk[(c0 + c) >> 1] = pack_bf16x2(p0, p1);
          }
        }
        rs = ((r8[0] + r8[1]) + (r8[2] + r8[3])) + ((r8[4] + r8[5]) + (r8[6] + r8[7]));
        l_sum = l_sum * alpha + rs;
        tmem_st32(s_col, pk);  // P over the first 64 columns of the S buffer
        tmem_st32(s_col + 32, pk + 32);
        // O_x must hold PV(v-1) before it is rescaled and before PV(v) adds to it
        if (v >= 1) {
          if (!__all_sync(0xffffffffu, mbar_wait_abortable(&o_done[x], (v - 1) & 1, 31, &s_abort))) {
            ok = false;
            break;
          }
          fence_after();
          if (__any_sync(0xffffffffu, grow)) {  // warp-uniform; rows that need none scale by 1
            const float f = grow ? alpha : 1.f;
#pragma unroll 1
            for (int c0 = 0; c0 < 128; c0 += 32) {
              float ov[32];
              tmem_ld32(o_col + c0, ov);
              wait_ld();
              uint32_t ou[32];
#pragma unroll
              for (int u = 0; u < 32; ++u) ou[u] = __float_as_uint(ov[u] * f);
              tmem_st32(o_col + c0, ou);
            }
          }
        }
      }
      wait_st();
      fence_before();
      __syncwarp();
      if (lane == 0) {
        if (!lo_sent) mbar_arrive(&p_lo[x]);
        mbar_arrive(&p_ready[x]);
      }
    }
    // epilogue: O / l -> bf16, LSE
    if (ok && nv > 0 && __all_sync(0xffffffffu, mbar_wait_abortable(&o_done[x], (nv - 1) & 1, 32, &s_abort))) {
      fence_after();
      const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
      const int rel = i - q_off;  // row of this query in the call's rows
      __nv_bfloat16* orow = a.out + ((static_cast<long long>(qrow0) + rel) * a.hq + h) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        float ov[32];
        tmem_ld32(o_col + c0, ov);
        wait_ld();
        if (rel < Lq) {
#pragma unroll
          for (int u = 0; u < 32; u += 8) {
            uint4 w;
            w.x = pack_bf16x2(ov[u] * inv, ov[u + 1] * inv);
            w.y = pack_bf16x2(ov[u + 2] * inv, ov[u + 3] * inv);
            w.z = pack_bf16x2(ov[u + 4] * inv, ov[u + 5] * inv);
            w.w = pack_bf16x2(ov[u + 6] * inv, ov[u + 7] * inv);
            *reinterpret_cast<uint4*>(orow + c0 + u) = w;
          }
        }
      }
      // Every valid row has at least one key in range, so its normaliser is finite and positive
      // unless an fp16 operand overflowed (an inf score makes the row NaN): report it.
      if (rel < Lq && !(l_sum > 0.f && l_sum < INFINITY && m_ref > -INFINITY && m_ref < INFINITY))
        report_status(kDevRange, 45);
      if (a.lse && rel < Lq) {
        // dense: [b, hq, Lq]; a paged batch: [hq, total_rows] over the packed rows
        const long long li = paged ? static_cast<long long>(h) * a.total_rows + qrow0 + rel
                                   : (static_cast<long long>(b) * a.hq + h) * a.Lq + rel;
        a.lse[li] = (m_ref + __log2f(l_sum)) * 0.69314718055994530942f;
      }
    }
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 9) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(NCOLS));
}

constexpr int attn_tc2_smem_bytes(bool fused = false) {
  return 2 * tc2::Q_BYTES + (fused ? tc2::NK3 + tc2::NV2 : tc2::NSLOT2) * tc::SLOT_BYTES;
}

}  // namespace bf
