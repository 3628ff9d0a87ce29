// RoPE and the correction rotation applied inside the prefill kernel's tile loads.
//
// In the fused form of the ping-pong prefill kernel, TMA brings RAW bf16 tiles (queries,
// raw keys, or cached keys) into the operand slots, and two transform warps rotate each
// tile in place into the fp16 QK^T operand the MMA reads, so no rotated copy of q or k
// exists in HBM (the on-the-fly rotation of the ai-feeds summary of Jet-Long, 方法 key
// module 3). Two key sources:
//   raw keys k_j (a prefill):             original form R(j w) k_j; long form R_long(j) k_j
//   cached keys kc_j = R(j w) k_j (bf16): original form kc_j as stored; long form
//                                         R_long(j) R(j w)^-1 kc_j, the correction rotation
// R_long is frequency interpolation (angle j w / G) or position aliasing (angle floor(j/G) w),
// the two long-range forms of the ablation in the same summary (实验). Pair k of the
// rotate-half layout is (d, d + 64), d = k, and both elements of a pair sit at the same
// offset of the two 128-byte-swizzled halves of a slot (d < 64 in the first 16 KB, d >= 64
// in the second), so the rotation needs no unswizzling.
//
// Thread layout (64 transform threads): thread pt owns chunk c = pt & 7 (pairs 8c .. 8c+7,
// 16 bytes of each half) and rows r0 + 8 m, r0 = pt >> 3 in 0..7, m = 0..15: every (row,
// chunk) of a 128-row tile once; the 32 lanes of a warp touch four whole 128-byte rows per
// access (no bank conflicts).
//
// Rotation angles of a key tile. An angle linear in the position, j * a_k, advances along a
// thread's rows by the fixed rotation R(8 a); after its 16 rows of a tile a thread stands at
// row r0 + 128, the first row of the next tile, so a run of consecutive tiles needs one exact
// angle per thread and pair (fp64 product and reduction, angle_cos_sin) and complex
// multiplications after that; the run is re-anchored every 8 tiles to bound the rounding
// drift (about 1e-7 per step). Position aliasing is linear in steps of G positions, so it
// takes the same path when G divides 8 (G = 1, 2, 4, 8); for any other G each row gets its
// exact angle. The arithmetic runs on packed fp32 pairs (two pairs per instruction).
//
// No per-element range check runs here (it would cost a fifth of the transform): an operand
// that fp16 cannot hold turns its scores into inf or NaN, and the kernel's epilogue reports
// any row whose softmax normaliser is not finite.
#pragma once
#include "common.cuh"

namespace bf {

struct RopeSrc {
  int cache;  // 1: the key tiles hold keys under the original RoPE (a cache), 0: raw keys
  int mode;   // 0 frequency interpolation, 1 position aliasing
  int G;      // the factor of a single sequence (a batch of sequences passes each one's own)
  double omega[64];  // omega_k = theta^(-2k/128)
};

namespace rl {
constexpr int FORM_ORIG = 0, FORM_LONG = 1;
constexpr int NXF = 64;  // transform threads
constexpr int ANCHOR_EVERY = 8;
}  // namespace rl

// Rotation of 8 pairs, two pairs per 64-bit register (the packed f32x2 arithmetic of sm_100):
// c[w] = (cos of pair 2w, cos of pair 2w+1), s[w] likewise.
struct Rot8 {
  uint64_t c[4], s[4];
};

// Angle of pair k at position j for the given form, in fp64; `key` selects the key source
// (queries are always raw).
__device__ __forceinline__ double rope_angle(const RopeSrc& s, int G, int form, bool key, long long j, int k) {
  const double om = s.omega[k];
  const bool cached = key && s.cache;
  if (form == rl::FORM_ORIG) return cached ? 0.0 : static_cast<double>(j) * om;
  if (s.mode == 0) return static_cast<double>(j) * (cached ? om / G - om : om / G);
  const double jg = static_cast<double>(j / G);
  return cached ? (jg - static_cast<double>(j)) * om : jg * om;
}

// Rate a_k of a form that is linear in the position (angle per position step).
__device__ __forceinline__ double rope_rate(const RopeSrc& s, int G, int form, bool key, int k) {
  const double om = s.omega[k];
  const bool cached = key && s.cache;
  if (form == rl::FORM_ORIG) return cached ? 0.0 : om;
  return cached ? om / G - om : om / G;
}

// Position aliasing advances by whole groups of G positions along 8-position steps only when G
// divides 8; every other form is linear in the position.
__device__ __forceinline__ bool form_linear(const RopeSrc& s, int G, int form) {
  return form == rl::FORM_ORIG || s.mode == 0 || (8 % G) == 0;
}

__device__ __forceinline__ void rot_exact(Rot8& R, const RopeSrc& s, int G, int form, bool key, long long j, int k0) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    float c0, s0, c1, s1;
    angle_cos_sin(rope_angle(s, G, form, key, j, k0 + 2 * w), c0, s0);
    angle_cos_sin(rope_angle(s, G, form, key, j, k0 + 2 * w + 1), c1, s1);
    R.c[w] = f2_pack(c0, c1);
    R.s[w] = f2_pack(s0, s1);
  }
}

__device__ __forceinline__ void rot_step(Rot8& R, const RopeSrc& s, int G, int form, bool key, int steps, int k0) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    float c0, s0, c1, s1;
    angle_cos_sin(static_cast<double>(steps) * rope_rate(s, G, form, key, k0 + 2 * w), c0, s0);
    angle_cos_sin(static_cast<double>(steps) * rope_rate(s, G, form, key, k0 + 2 * w + 1), c1, s1);
    R.c[w] = f2_pack(c0, c1);
    R.s[w] = f2_pack(s0, s1);
  }
}

// R <- R * S (angles add): (c, s) -> (c cS - s sS, s cS + c sS)
__device__ __forceinline__ void rot_mul(Rot8& R, const Rot8& S) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const uint64_t c = f2_sub(f2_mul(R.c[w], S.c[w]), f2_mul(R.s[w], S.s[w]));
    R.s[w] = f2_fma(R.c[w], S.s[w], f2_mul(R.s[w], S.c[w]));
    R.c[w] = c;
  }
}

__device__ __forceinline__ uint4 ld_shared16(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
  return r;
}
__device__ __forceinline__ void st_shared16(uint32_t addr, const uint4& v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// Two bf16 of one word as a packed pair of fp32 (a bf16 is the high half of its fp32).

// 8 pairs: x = elements 8c..8c+7 (bf16, in a), y = their partners 64 later (bf16, in b).
// (x, y) -> (x cos - y sin, y cos + x sin), rounded to fp16, written back over a and b.
__device__ __forceinline__ void rotate8(uint4& a, uint4& b, const Rot8& R) {
  uint32_t* wa = &a.x;
  uint32_t* wb = &b.x;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const uint64_t x = bf16x2_to_f2(wa[w]), y = bf16x2_to_f2(wb[w]);
    wa[w] = f2_to_f16x2(f2_sub(f2_mul(x, R.c[w]), f2_mul(y, R.s[w])));
    wb[w] = f2_to_f16x2(f2_fma(x, R.s[w], f2_mul(y, R.c[w])));
  }
}

// bf16 -> fp16 without rotation (cached keys in their original form)
__device__ __forceinline__ void convert8(uint4& a, uint4& b) {
  uint32_t* wa = &a.x;
  uint32_t* wb = &b.x;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    wa[w] = f2_to_f16x2(bf16x2_to_f2(wa[w]));
    wb[w] = f2_to_f16x2(bf16x2_to_f2(wb[w]));
  }
}

// Swizzled byte offset of (row r, 16-byte chunk c) in one 128-row x 128-byte half of a slot.
__device__ __forceinline__ uint32_t slot_off(int r, int c) { return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4)); }

// Rotates, in place, the key tile of keys j0 .. j0+127 held raw in the slot at shared
// address `slot` into form `form`. Rows of keys >= Lk (past the sequence: zero-filled by the
// copy, or whatever a paged pool holds there) are written as zeros. `st` holds this thread's
// rotation at key j0 + r0 on entry (linear forms) and at j0 + 128 + r0 on return; `s8` is the
// rotation of 8 positions.
__device__ __forceinline__ void rope_key_tile(uint32_t slot, const RopeSrc& s, int G, int form, bool linear, int j0,
                                              int Lk, int cch, int r0, Rot8& st, const Rot8& s8) {
  const bool ident = s.cache && form == rl::FORM_ORIG;
  if (ident || linear) {
#pragma unroll 2
    for (int m = 0; m < 16; ++m) {
      const int r = r0 + 8 * m;
      const uint32_t off = slot + slot_off(r, cch);
      uint4 a = make_uint4(0u, 0u, 0u, 0u), b = a;
      if (j0 + r < Lk) {
        a = ld_shared16(off);
        b = ld_shared16(off + 16384);
        if (ident)
          convert8(a, b);
        else
          rotate8(a, b, st);
      }
      if (!ident) rot_mul(st, s8);
      st_shared16(off, a);
      st_shared16(off + 16384, b);
    }
  } else {
    // position aliasing with a G that does not divide 8: an exact angle per row
#pragma unroll 1
    for (int m = 0; m < 16; ++m) {
      const int r = r0 + 8 * m;
      const uint32_t off = slot + slot_off(r, cch);
      uint4 a = make_uint4(0u, 0u, 0u, 0u), b = a;
      if (j0 + r < Lk) {
        a = ld_shared16(off);
        b = ld_shared16(off + 16384);
        Rot8 R;
        rot_exact(R, s, G, form, true, j0 + r, 8 * cch);
        rotate8(a, b, R);
      }
      st_shared16(off, a);
      st_shared16(off + 16384, b);
    }
  }
}

// Zeroes the rows r_lo .. 127 of a V tile (both halves): the keys past a sequence's end in a
// paged pool, whose P is 0 but whose values may be anything (0 * NaN would be NaN).
__device__ __forceinline__ void zero_tile_rows(uint32_t slot, int r_lo, int cch, int r0) {
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll 1
  for (int m = 0; m < 16; ++m) {
    const int r = r0 + 8 * m;
    if (r >= r_lo) {
      st_shared16(slot + slot_off(r, cch), z);
      st_shared16(slot + 16384 + slot_off(r, cch), z);
    }
  }
}

// Rotates, in place, the raw query tiles of two heads (Q_A at qslot, Q_B 32 KB above) of
// rows at absolute positions i0 .. i0+127 into form `form`, with the same incremental angles
// as the key tiles (one exact angle per thread and pair, then 8-position steps) where the form
// is linear, else an exact angle per row.
__device__ __forceinline__ void rope_query_tiles(uint32_t qslot, const RopeSrc& s, int G, int form, int i0, int cch,
                                                 int r0) {
  const bool linear = form_linear(s, G, form);
  Rot8 R, s8;
  rot_exact(R, s, G, form, false, i0 + r0, 8 * cch);
  if (linear) rot_step(s8, s, G, form, false, 8, 8 * cch);
#pragma unroll 1
  for (int m = 0; m < 16; ++m) {
    const int r = r0 + 8 * m;
    if (!linear && m > 0) rot_exact(R, s, G, form, false, i0 + r, 8 * cch);
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const uint32_t off = qslot + x * 32768 + slot_off(r, cch);
      uint4 a = ld_shared16(off), b = ld_shared16(off + 16384);
      rotate8(a, b, R);
      st_shared16(off, a);
      st_shared16(off + 16384, b);
    }
    if (linear) rot_mul(R, s8);
  }
}

}  // namespace bf
