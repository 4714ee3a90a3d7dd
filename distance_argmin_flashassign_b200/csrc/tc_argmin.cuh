// tc_argmin.cuh -- the arg-max epilogue shared by the tensor-core
// assignment kernels: each thread holds one point's row of scores
// s_k = <x, c_k> - |c_k|^2 / 2 in 32-column chunks read from TMEM, keeps the
// running best (lowest column on ties) and the runner-up information the
// exact re-decision needs, and lists the points it cannot order with
// certainty.
#pragma once
#include "fk_internal.h"

namespace fk {

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Maximum of 32 scores: four interleaved chains of 3-input max over eight
// values each (few live temporaries), then their maximum.
__device__ __forceinline__ float max32(const uint32_t (&v)[32]) {
  float m[4];
#pragma unroll
  for (int c = 0; c < 4; ++c)
    m[c] = fmax3(__uint_as_float(v[8 * c]), __uint_as_float(v[8 * c + 1]), __uint_as_float(v[8 * c + 2]));
#pragma unroll
  for (int c = 0; c < 4; ++c) m[c] = fmax3(m[c], __uint_as_float(v[8 * c + 3]), __uint_as_float(v[8 * c + 4]));
#pragma unroll
  for (int c = 0; c < 4; ++c) m[c] = fmax3(m[c], __uint_as_float(v[8 * c + 5]), __uint_as_float(v[8 * c + 6]));
#pragma unroll
  for (int c = 0; c < 4; ++c) m[c] = fmaxf(m[c], __uint_as_float(v[8 * c + 7]));
  return fmaxf(fmax3(m[0], m[1], m[2]), m[3]);
}


// Running arg-max of one point over the chunks it has seen, in column order,
// and the two best maxima of the other chunks (the runner-up chunk's, with
// its first column, and the third chunk's).
struct Best {
  float score;
  int base;           // first column of the candidate chunk
  float s2;           // largest chunk maximum among the other chunks
  int base2;          // first column of the chunk holding s2 (-1: none yet)
  float s3;           // second largest chunk maximum among the other chunks
  uint32_t cand[32];  // the chunk that first reached `score`
};

// Leave column e of a chunk out (its score becomes -inf), for e in [0, 32).
__device__ __forceinline__ void mask_col(uint32_t (&v)[32], int e) {
  if ((unsigned)e < 32u) {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i == e) v[i] = 0xff800000u;
  }
}

__device__ __forceinline__ void best_init(Best &bs) {
  bs.score = __int_as_float(0xff800000);
  bs.base = 0;
  bs.s2 = __int_as_float(0xff800000);
  bs.base2 = -1;
  bs.s3 = __int_as_float(0xff800000);
#pragma unroll
  for (int i = 0; i < 32; ++i) bs.cand[i] = 0u;
}

// (d0, d1) = (a0 + b0, a1 + b1) in one packed fp32 add (FMA pipe).
__device__ __forceinline__ void add2(uint32_t &d0, uint32_t &d1, uint32_t a0, uint32_t a1, uint32_t b0,
                                     uint32_t b1) {
  asm("{\n\t.reg .b64 x, y, z;\n\tmov.b64 x, {%2, %3};\n\tmov.b64 y, {%4, %5};\n\t"
      "add.rn.f32x2 z, x, y;\n\tmov.b64 {%0, %1}, z;\n\t}"
      : "=r"(d0), "=r"(d1)
      : "r"(a0), "r"(a1), "r"(b0), "r"(b1));
}

// (a0, a1) += (v0 * v0, v1 * v1) in one packed fp32 fma.
__device__ __forceinline__ void fma2(uint32_t &a0, uint32_t &a1, uint32_t v0, uint32_t v1) {
  asm("{\n\t.reg .b64 a, v;\n\tmov.b64 a, {%0, %1};\n\tmov.b64 v, {%2, %3};\n\t"
      "fma.rn.f32x2 a, v, v, a;\n\tmov.b64 {%0, %1}, a;\n\t}"
      : "+r"(a0), "+r"(a1)
      : "r"(v0), "r"(v1));
}

// Fold one 32-column chunk of scores (first column `col`) into the running
// arg-max.  The candidate copy is written as x + 0 (packed add.rn.f32x2, two
// values per instruction on the FMA pipe, leaving the half-rate logic pipe
// to the max trees); it keeps every value but turns -0 into +0, which
// compares equal, so the index search below finds the same column.
//
// The chunk that does not hold the running maximum after the fold (the new
// chunk, or the previous holder when the new chunk beats it) competes for
// the runner-up chunk: its maximum min(m, score) replaces s2 when larger,
// and the smaller of the two competes for s3.
__device__ __forceinline__ void fold_chunk(Best &bs, const uint32_t (&v)[32], int col) {
  const float m = max32(v);
  const bool imp = m > bs.score;  // strict: an earlier column keeps a tie
  const float lo = fminf(m, bs.score);
  const int lob = imp ? bs.base : col;
  bs.s3 = fmaxf(bs.s3, fminf(lo, bs.s2));
  const bool up = lo > bs.s2;
  bs.s2 = up ? lo : bs.s2;
  bs.base2 = up ? lob : bs.base2;
  if (__any_sync(0xffffffffu, imp)) {
    if (imp) {
#pragma unroll
      for (int i = 0; i < 32; i += 2) add2(bs.cand[i], bs.cand[i + 1], v[i], v[i + 1], 0u, 0u);
      bs.score = m;
      bs.base = col;
    }
  }
}

// Largest score of the candidate chunk other than the one at position jm.
__device__ __forceinline__ float second_in_chunk(const Best &bs, int jm) {
  float m[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) m[c] = __int_as_float(0xff800000);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float v = i == jm ? __int_as_float(0xff800000) : __uint_as_float(bs.cand[i]);
    m[i & 3] = fmaxf(m[i & 3], v);
  }
  return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// A point whose best score s1 and runner-up s2 differ by no more than the
// fp32 rounding of the scores may be ordered wrongly: it is listed for the
// exact re-decision (refine.cu) together with the first column of the other
// chunk it must re-examine, or for a comparison with every centroid when
// the best maximum of a third chunk, s3, is that close too.  |x|^2 + |c_best|^2 <= 5|x|^2 - 4 s1
// (as |c| <= |x| + |x - c| and |x - c|^2 = |x|^2 - 2 s1) bounds the
// magnitudes the scores are accumulated from.  The warp appends its listed
// points with one atomic add.
__device__ __forceinline__ void list_near_tie(const NearTies &t, bool valid, float s1, float s2, float s3,
                                              float xn, size_t g, int other) {
  if (t.list == nullptr) return;
  const float thr = t.tau * fmaxf(5.f * xn - 4.f * s1, 0.f);
  const bool near = valid && (s1 - s2) <= thr;
  list_append(t, near, (s1 - s3) <= thr, (int)g, other);
}


// Position (0-31) of the lowest column of the candidate chunk holding the
// maximum, 32 if none does.
__device__ __forceinline__ int best_pos(const Best &bs) {
  int j0 = 32, j1 = 32, j2 = 32, j3 = 32;
#pragma unroll
  for (int i = 28; i >= 0; i -= 4) {
    j0 = __uint_as_float(bs.cand[i]) == bs.score ? i : j0;
    j1 = __uint_as_float(bs.cand[i + 1]) == bs.score ? i + 1 : j1;
    j2 = __uint_as_float(bs.cand[i + 2]) == bs.score ? i + 2 : j2;
    j3 = __uint_as_float(bs.cand[i + 3]) == bs.score ? i + 3 : j3;
  }
  return min(min(j0, j1), min(j2, j3));
}

}  // namespace fk
