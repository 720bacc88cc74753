// Device side of the gated delta rule decode library (sm_100a).
//
// The decode step is HBM-bound: per (sequence, head) the dk x dv fp32 state
// is read once and written once, and the arithmetic is two mat-vec products
// and a rank-1 update (about 7 flop per 8 bytes of state), so there is no
// dense contraction for the tensor cores.  The kernels below are built as a
// stream over state rows:
//
//   * A state row is one dv column of S: dk contiguous floats (512 B for
//     dk = 128).  A warp is split into groups of LPR lanes; each group owns
//     M consecutive rows and each lane holds EL = dk/LPR elements of every
//     row of its group, as 4-float chunks placed so that one warp-wide
//     128-bit load or store moves LPR*16 contiguous bytes of each of the
//     32/LPR rows in flight (full 128-byte lines for LPR >= 8).
//   * Per token, both dot products S^T k and S^T q of every row, plus the
//     three scalars |k|^2, |q|^2 and k.q needed for the L2 norms, are summed
//     in ONE xor butterfly over the LPR lanes of a group: log2(LPR) shuffle
//     levels, after which every lane of the group holds every sum with the
//     same bits.
//   * The read-out uses the updated state without a second pass over it:
//       o_j = scale * (alpha (S^T q)_j + (k.q) delta_j)
//     which is S'^T q for S' = alpha S + k delta^T, exactly in real
//     arithmetic.
//   * The state stays in registers across the T tokens of a call, so HBM
//     traffic does not depend on T.
//   * The token arithmetic uses explicitly rounded intrinsics
//     (__fmul_rn/__fmaf_rn/__fadd_rn) so that the compiler cannot contract it
//     differently in different instantiations: in decode_kernel a T-token
//     call is bit-identical to T one-token calls.  decode_block_smem_kernel
//     (calls of 2..4 tokens on fp32 pools) unrolls the recurrence over the
//     call's tokens instead; its first token carries the one-token bits, the
//     later ones agree with the token-by-token order to fp32 rounding, and a
//     call that stores the state after n tokens carries the bits of an
//     n-token call.
//   * Each CTA also asks L2 for the state tile of the CTA up to one wave of
//     resident CTAs later, so the state stream keeps bytes in flight while
//     the resident CTAs compute.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------------------
// division by a divisor fixed at launch
//
// A CTA finds its (sequence, head, tile) from its block index by dividing by
// the head count and the tiles per head, and its k head by dividing by the
// GQA group: with the divisors known only at run time, each is a sequence
// of a few dozen instructions, a measurable share of a short CTA's work.
// The host instead computes, once per launch, l = ceil(log2 d) and
// m = floor(2^32 (2^l - d) / d) + 1 (less than 2^32); then for 0 <= n < 2^31,
// floor(n / d) = (umulhi(n, m) + n) >> l (Granlund and Montgomery, "Division
// by invariant integers using multiplication", PLDI 1994, theorem 4.2 with
// N = 32; n < 2^31 keeps the sum within 32 bits).
struct FastDiv {
  uint32_t d, m, l;
};

__host__ inline FastDiv make_fast_div(uint32_t d) {
  FastDiv f{d, 1u, 0u};
  if (d == 0) return f;  // no kernel divides by it (an empty dimension launches nothing)
  while ((1ull << f.l) < d) ++f.l;
  f.m = (uint32_t)((((1ull << 32) * ((1ull << f.l) - d)) / d) + 1);
  return f;
}

// floor(n / f.d) for 0 <= n < 2^31
__device__ __forceinline__ int fdiv(int n, const FastDiv& f) {
  return (int)((__umulhi((uint32_t)n, f.m) + (uint32_t)n) >> f.l);
}

// ---------------------------------------------------------------------------
// raw vector loads and stores

template <int BYTES>
struct RawVec;
template <>
struct RawVec<2> {
  static constexpr int W = 1;
};
template <>
struct RawVec<4> {
  static constexpr int W = 1;
};
template <>
struct RawVec<8> {
  static constexpr int W = 2;
};
template <>
struct RawVec<16> {
  static constexpr int W = 4;
};
template <>
struct RawVec<32> {
  static constexpr int W = 8;
};
template <>
struct RawVec<64> {
  static constexpr int W = 16;
};

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t u16) {
  return __uint_as_float(u16 << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float x) {
  __nv_bfloat16 h = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&h);
}

// Load N consecutive elements of type In (float or __nv_bfloat16) from p,
// which is aligned to N * sizeof(In) bytes, converting to float.
template <typename In, int N>
__device__ __forceinline__ void load_vec(const In* p, float (&o)[N]) {
  constexpr int BYTES = N * (int)sizeof(In);
  uint32_t w[RawVec<BYTES>::W];
  if constexpr (BYTES == 2) {
    w[0] = *reinterpret_cast<const uint16_t*>(p);
  } else if constexpr (BYTES == 4) {
    w[0] = *reinterpret_cast<const uint32_t*>(p);
  } else if constexpr (BYTES == 8) {
    uint2 t = *reinterpret_cast<const uint2*>(p);
    w[0] = t.x;
    w[1] = t.y;
  } else if constexpr (BYTES == 16) {
    uint4 t = *reinterpret_cast<const uint4*>(p);
    w[0] = t.x;
    w[1] = t.y;
    w[2] = t.z;
    w[3] = t.w;
  } else {
    static_assert(BYTES == 32 || BYTES == 64, "unsupported vector size");
#pragma unroll
    for (int c = 0; c < BYTES / 16; ++c) {
      const uint4 t = reinterpret_cast<const uint4*>(p)[c];
      w[4 * c + 0] = t.x;
      w[4 * c + 1] = t.y;
      w[4 * c + 2] = t.z;
      w[4 * c + 3] = t.w;
    }
  }
  if constexpr (sizeof(In) == 4) {
#pragma unroll
    for (int i = 0; i < N; ++i) o[i] = __uint_as_float(w[i]);
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      uint32_t word = w[i / 2];
      o[i] = bf16_bits_to_f32((i & 1) ? (word >> 16) : (word & 0xffffu));
    }
  }
}

template <typename Out>
__device__ __forceinline__ void store_scalar(Out* p, float x) {
  if constexpr (sizeof(Out) == 4) {
    *reinterpret_cast<float*>(p) = x;
  } else {
    *reinterpret_cast<uint16_t*>(p) = f32_to_bf16_bits(x);
  }
}

// ---------------------------------------------------------------------------
// lane groups over state rows

// Placement of one row's dk elements over the LPR lanes of a group: lane
// position pos = lane % LPR holds chunks c = 0..CH-1 of CW elements, chunk c
// covering dk indices [CW*(pos + LPR*c), CW*(pos + LPR*c) + CW).  A chunk is
// 16 bytes of state (CW = 4 fp32 or 8 bf16/fp16 values), so one warp-wide
// load of chunk c moves LPR*16 contiguous bytes of each of 32/LPR rows.
template <int DK, int LPR, int CW>
struct Lanes {
  static_assert(LPR == 4 || LPR == 8 || LPR == 16 || LPR == 32, "LPR must divide 32");
  static constexpr int EL = DK / LPR;   // elements of a row per lane
  static constexpr int CH = EL / CW;    // chunks per lane
  static constexpr int GROUPS = 32 / LPR;
  static_assert(EL % CW == 0, "a lane holds whole chunks");
  __device__ static __forceinline__ int offset(int pos, int c) { return CW * (pos + LPR * c); }
};

template <typename St>
struct StateTraits;
template <>
struct StateTraits<float> {
  static constexpr int CW = 4;
};
template <>
struct StateTraits<__nv_bfloat16> {
  static constexpr int CW = 8;
};
template <>
struct StateTraits<__half> {
  static constexpr int CW = 8;
};

__device__ __forceinline__ uint32_t pack2(__nv_bfloat16, float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack2(__half, float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ void unpack2(__nv_bfloat16, uint32_t w, float& a, float& b) {
  a = __uint_as_float(w << 16);
  b = __uint_as_float(w & 0xffff0000u);
}
__device__ __forceinline__ void unpack2(__half, uint32_t w, float& a, float& b) {
  const __half2 h = *reinterpret_cast<const __half2*>(&w);
  const float2 f = __half22float2(h);
  a = f.x;
  b = f.y;
}

// One row of the state, converted to fp32 (streaming hints: the state is
// touched once per call, so it should not displace the small per-token
// inputs in L2).  16-bit states are rounded to nearest-even on the way out.
template <typename St, int DK, int LPR>
__device__ __forceinline__ void load_row(const St* row, int pos, float (&s)[DK / LPR]) {
  using L = Lanes<DK, LPR, StateTraits<St>::CW>;
#pragma unroll
  for (int c = 0; c < L::CH; ++c) {
    if constexpr (sizeof(St) == 4) {
      const float4 t = __ldcs(reinterpret_cast<const float4*>(row + L::offset(pos, c)));
      s[4 * c + 0] = t.x;
      s[4 * c + 1] = t.y;
      s[4 * c + 2] = t.z;
      s[4 * c + 3] = t.w;
    } else {
      const uint4 t = __ldcs(reinterpret_cast<const uint4*>(row + L::offset(pos, c)));
      unpack2(St(), t.x, s[8 * c + 0], s[8 * c + 1]);
      unpack2(St(), t.y, s[8 * c + 2], s[8 * c + 3]);
      unpack2(St(), t.z, s[8 * c + 4], s[8 * c + 5]);
      unpack2(St(), t.w, s[8 * c + 6], s[8 * c + 7]);
    }
  }
}

template <typename St, int DK, int LPR>
__device__ __forceinline__ void store_row(St* row, int pos, const float (&s)[DK / LPR]) {
  using L = Lanes<DK, LPR, StateTraits<St>::CW>;
#pragma unroll
  for (int c = 0; c < L::CH; ++c) {
    if constexpr (sizeof(St) == 4) {
      __stcs(reinterpret_cast<float4*>(row + L::offset(pos, c)),
             make_float4(s[4 * c + 0], s[4 * c + 1], s[4 * c + 2], s[4 * c + 3]));
    } else {
      uint4 t;
      t.x = pack2(St(), s[8 * c + 0], s[8 * c + 1]);
      t.y = pack2(St(), s[8 * c + 2], s[8 * c + 3]);
      t.z = pack2(St(), s[8 * c + 4], s[8 * c + 5]);
      t.w = pack2(St(), s[8 * c + 6], s[8 * c + 7]);
      __stcs(reinterpret_cast<uint4*>(row + L::offset(pos, c)), t);
    }
  }
}

// All-reduce N values over each aligned group of LPR lanes (xor butterfly).
// Every lane of a group ends with the same bits: each partner pair adds the
// same two operands.
template <int LPR, int N>
__device__ __forceinline__ void group_allreduce(float (&x)[N]) {
#pragma unroll
  for (int off = LPR / 2; off >= 1; off >>= 1) {
#pragma unroll
    for (int i = 0; i < N; ++i) x[i] = __fadd_rn(x[i], __shfl_xor_sync(kFull, x[i], off));
  }
}

// ---------------------------------------------------------------------------
// one token on the M rows of a lane group

struct TokenScalars {
  float alpha;  // exp(g)
  float beta;
  float scale;
  float kq;     // k_hat . q_hat
};

// Apply one token to the group's M rows S[m][0..EL) (this lane's elements)
// and return their outputs o_m (identical in every lane of the group).
//   kn, qn : this lane's elements of the normalised k and q
//   vv     : v_j of the group's M rows
// delta_j = beta (v_j - alpha (S^T k)_j);  o_j = scale (alpha (S^T q)_j +
// (k.q) delta_j);  S_ij <- alpha S_ij + k_i delta_j.
// Paired fp32 arithmetic (sm_100): a 64-bit register holds two floats, the
// first in the low half; each half is rounded as the scalar operation.
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void split_f32x2(uint64_t r, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

template <int LPR, int EL, int M, bool PAIRED = true>
__device__ __forceinline__ void token_rows(float (&S)[M][EL], const float (&kn)[EL],
                                           const float (&qn)[EL], const float (&vv)[M],
                                           const TokenScalars& ts, float (&o)[M]) {
  float red[2 * M];  // [m] = S_m . k,  [M+m] = S_m . q
#pragma unroll
  for (int m = 0; m < M; ++m) {
    float pk = __fmul_rn(S[m][0], kn[0]);
    float pq = __fmul_rn(S[m][0], qn[0]);
#pragma unroll
    for (int e = 1; e < EL; ++e) {
      pk = __fmaf_rn(S[m][e], kn[e], pk);
      pq = __fmaf_rn(S[m][e], qn[e], pq);
    }
    red[m] = pk;
    red[M + m] = pq;
  }
  group_allreduce<LPR, 2 * M>(red);
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const float d = __fmul_rn(ts.beta, __fsub_rn(vv[m], __fmul_rn(ts.alpha, red[m])));
    o[m] = __fmul_rn(ts.scale, __fmaf_rn(ts.kq, d, __fmul_rn(ts.alpha, red[M + m])));
    if constexpr (PAIRED && EL % 2 == 0) {
      // in paired fp32 arithmetic, two elements per instruction, same bits
      // (it shortens the arithmetic-bound token loop; the fused kernel, which
      // measured a hair slower with it, keeps the scalar form)
      const uint64_t a2 = f32x2(ts.alpha, ts.alpha), d2 = f32x2(d, d);
#pragma unroll
      for (int e = 0; e < EL; e += 2)
        split_f32x2(fma_f32x2(f32x2(kn[e], kn[e + 1]), d2,
                              mul_f32x2(a2, f32x2(S[m][e], S[m][e + 1]))),
                    S[m][e], S[m][e + 1]);
    } else {
#pragma unroll
      for (int e = 0; e < EL; ++e) S[m][e] = __fmaf_rn(kn[e], d, __fmul_rn(ts.alpha, S[m][e]));
    }
  }
}

// The same token on rows kept packed as pairs of 16-bit values (St = bf16 or
// fp16): each pair is widened to fp32 where it is used, the update is
// computed in fp32 as in token_rows and rounded to nearest-even when it is
// packed again.  The loops run chunk by chunk and read the normalised k and
// q from shared memory per chunk, so only the packed rows stay in registers.
// Only valid for single-token calls (the packed rows hold the rounded state).
template <typename St, int DK, int LPR, int M>
__device__ __forceinline__ void token_rows_packed(uint32_t (&P)[M][DK / LPR / 2],
                                                  const float* kn_s, const float* qn_s, int pos,
                                                  const float (&vv)[M], const TokenScalars& ts,
                                                  float (&o)[M]) {
  using L = Lanes<DK, LPR, 8>;
  float red[2 * M];  // [m] = S_m . k,  [M+m] = S_m . q
#pragma unroll
  for (int m = 0; m < 2 * M; ++m) red[m] = 0.0f;
#pragma unroll
  for (int c = 0; c < L::CH; ++c) {
    float kc[8], qc[8];
    const float4 k0 = *reinterpret_cast<const float4*>(kn_s + L::offset(pos, c));
    const float4 k1 = *reinterpret_cast<const float4*>(kn_s + L::offset(pos, c) + 4);
    const float4 q0 = *reinterpret_cast<const float4*>(qn_s + L::offset(pos, c));
    const float4 q1 = *reinterpret_cast<const float4*>(qn_s + L::offset(pos, c) + 4);
    kc[0] = k0.x; kc[1] = k0.y; kc[2] = k0.z; kc[3] = k0.w;
    kc[4] = k1.x; kc[5] = k1.y; kc[6] = k1.z; kc[7] = k1.w;
    qc[0] = q0.x; qc[1] = q0.y; qc[2] = q0.z; qc[3] = q0.w;
    qc[4] = q1.x; qc[5] = q1.y; qc[6] = q1.z; qc[7] = q1.w;
#pragma unroll
    for (int m = 0; m < M; ++m) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float s0, s1;
        unpack2(St(), P[m][4 * c + i], s0, s1);
        red[m] = __fmaf_rn(s0, kc[2 * i], red[m]);
        red[M + m] = __fmaf_rn(s0, qc[2 * i], red[M + m]);
        red[m] = __fmaf_rn(s1, kc[2 * i + 1], red[m]);
        red[M + m] = __fmaf_rn(s1, qc[2 * i + 1], red[M + m]);
      }
    }
  }
  // Keep only the packed words live across the reduction: the empty asm
  // makes the widened values of the first pass unusable below, so they are
  // widened again instead of being held in twice the registers.
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int i = 0; i < DK / LPR / 2; ++i) asm volatile("" : "+r"(P[m][i]));
  group_allreduce<LPR, 2 * M>(red);
  float d[M];
#pragma unroll
  for (int m = 0; m < M; ++m) {
    d[m] = __fmul_rn(ts.beta, __fsub_rn(vv[m], __fmul_rn(ts.alpha, red[m])));
    o[m] = __fmul_rn(ts.scale, __fmaf_rn(ts.kq, d[m], __fmul_rn(ts.alpha, red[M + m])));
  }
  // the update in paired fp32 arithmetic: each half of mul.rn.f32x2 /
  // fma.rn.f32x2 is rounded as the scalar operation, so the bits are those of
  // fma(k, d, alpha * s) element by element
  const uint64_t a2 = f32x2(ts.alpha, ts.alpha);
  uint64_t d2[M];
#pragma unroll
  for (int m = 0; m < M; ++m) d2[m] = f32x2(d[m], d[m]);
#pragma unroll
  for (int c = 0; c < L::CH; ++c) {
    const float4 k0 = *reinterpret_cast<const float4*>(kn_s + L::offset(pos, c));
    const float4 k1 = *reinterpret_cast<const float4*>(kn_s + L::offset(pos, c) + 4);
    const uint64_t kc2[4] = {f32x2(k0.x, k0.y), f32x2(k0.z, k0.w), f32x2(k1.x, k1.y),
                             f32x2(k1.z, k1.w)};
#pragma unroll
    for (int m = 0; m < M; ++m) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float s0, s1;
        unpack2(St(), P[m][4 * c + i], s0, s1);
        const uint64_t y = fma_f32x2(kc2[i], d2[m], mul_f32x2(a2, f32x2(s0, s1)));
        float y0, y1;
        split_f32x2(y, y0, y1);
        P[m][4 * c + i] = pack2(St(), y0, y1);
      }
    }
  }
}

// Normalise one token's q and k (dk elements of type In) with one warp:
// lane l takes elements [l*DK/32, (l+1)*DK/32); |k|^2, |q|^2 and k.q are
// summed in one butterfly; k_hat = k / sqrt(|k|^2 + eps) (likewise q) go to
// shared memory with k_hat . q_hat.  Without l2norm the vectors are copied.
template <int DK>
__device__ __forceinline__ void normalise_loaded(float (&kv)[DK / 32], float (&qv)[DK / 32],
                                                 int lane, float eps, int l2norm, float* kn_s,
                                                 float* qn_s, float* kq_s);

template <typename In, int DK>
__device__ __forceinline__ void normalise_qk(const In* k, const In* q, int lane, float eps,
                                             int l2norm, float* kn_s, float* qn_s, float* kq_s) {
  constexpr int E = DK / 32;
  float kv[E], qv[E];
  load_vec<In, E>(k + lane * E, kv);
  load_vec<In, E>(q + lane * E, qv);
  normalise_loaded<DK>(kv, qv, lane, eps, l2norm, kn_s, qn_s, kq_s);
}

// The arithmetic of normalise_qk on this lane's elements, already loaded
// (so that a kernel can issue the loads early).
template <int DK>
__device__ __forceinline__ void normalise_loaded(float (&kv)[DK / 32], float (&qv)[DK / 32],
                                                 int lane, float eps, int l2norm, float* kn_s,
                                                 float* qn_s, float* kq_s) {
  constexpr int E = DK / 32;
  float red[3];
  red[0] = __fmul_rn(kv[0], kv[0]);
  red[1] = __fmul_rn(qv[0], qv[0]);
  red[2] = __fmul_rn(kv[0], qv[0]);
#pragma unroll
  for (int e = 1; e < E; ++e) {
    red[0] = __fmaf_rn(kv[e], kv[e], red[0]);
    red[1] = __fmaf_rn(qv[e], qv[e], red[1]);
    red[2] = __fmaf_rn(kv[e], qv[e], red[2]);
  }
  group_allreduce<32, 3>(red);
  float rk = 1.0f, rq = 1.0f;
  if (l2norm) {
    rk = rsqrtf(__fadd_rn(red[0], eps));
    rq = rsqrtf(__fadd_rn(red[1], eps));
  }
#pragma unroll
  for (int e = 0; e < E; ++e) {
    kv[e] = __fmul_rn(kv[e], rk);
    qv[e] = __fmul_rn(qv[e], rq);
  }
  // one vector store per lane and vector (kn_s and qn_s are 16-byte aligned):
  // consecutive lanes fill consecutive bytes, with no bank conflict
  if constexpr (E == 4) {
    *reinterpret_cast<float4*>(kn_s + lane * E) = make_float4(kv[0], kv[1], kv[2], kv[3]);
    *reinterpret_cast<float4*>(qn_s + lane * E) = make_float4(qv[0], qv[1], qv[2], qv[3]);
  } else if constexpr (E == 2) {
    *reinterpret_cast<float2*>(kn_s + lane * E) = make_float2(kv[0], kv[1]);
    *reinterpret_cast<float2*>(qn_s + lane * E) = make_float2(qv[0], qv[1]);
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      kn_s[lane * E + e] = kv[e];
      qn_s[lane * E + e] = qv[e];
    }
  }
  if (lane == 0) *kq_s = __fmul_rn(__fmul_rn(red[2], rk), rq);
}

// This lane's elements (placement of Lanes<DK, LPR, CW>) of a normalised
// vector held in shared memory.
template <int DK, int LPR, int CW>
__device__ __forceinline__ void lanes_from_smem(const float* v, int pos, float (&x)[DK / LPR]) {
  using L = Lanes<DK, LPR, CW>;
#pragma unroll
  for (int c = 0; c < L::CH; ++c) {
#pragma unroll
    for (int i = 0; i < CW; i += 4) {
      const float4 t = *reinterpret_cast<const float4*>(v + L::offset(pos, c) + i);
      x[CW * c + i + 0] = t.x;
      x[CW * c + i + 1] = t.y;
      x[CW * c + i + 2] = t.z;
      x[CW * c + i + 3] = t.w;
    }
  }
}

// the lane at group position m (< M) picks o[m]; other lanes get o[0]
template <int M>
__device__ __forceinline__ float select_row(const float (&o)[M], int pos) {
  float x = o[0];
#pragma unroll
  for (int m = 1; m < M; ++m) x = (pos == m) ? o[m] : x;
  return x;
}

// ---------------------------------------------------------------------------
// the batched decode step

struct StepParams {
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const float* beta;
  void* state;  // [n_slots][H][dv][dk] of the state type
  const int32_t* slot_idx;
  void* out;
  int B, Hk, H, dv, T, n_slots, group;
  float scale, l2_eps;
  int l2norm;
  int* dev_status;
  const int32_t* n_accept;     // [B] or null: commit the state after n_accept[b] tokens
  const int32_t* token_slots;  // [B][T] or null: store the state after token t there
  int prefetch_ahead;          // > 0: each CTA asks L2 for the tile of CTA blockIdx + this
  FastDiv div_h, div_group, div_tiles;  // by H, by group, by tiles per head (set at launch)
};

// L2 prefetch of `bytes` (a multiple of 16, 16-byte aligned) of global memory:
// one bulk request with no completion to wait for.
__device__ __forceinline__ void prefetch_l2(const void* src, unsigned bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(src), "r"(bytes) : "memory");
}

// L2 prefetch of the cache line holding `src` (any alignment).
__device__ __forceinline__ void prefetch_l2_line(const void* src) {
  asm volatile("prefetch.global.L2 [%0];\n" ::"l"(src) : "memory");
}

// The state stream keeps a resident CTA's bytes in flight only until its
// tile has landed; the rest of its life is arithmetic.  So a CTA also
// requests, into L2, the tile of the CTA `prefetch_ahead` launches later
// (up to one wave of resident CTAs on), whose own loads then hit L2.  Grid
// order as decode_kernel: tile fastest, then h, then b.  In two halves, so
// that the warp which issues it never waits for the future CTA's slot:
// future_tile_begin issues the load of that slot (s = -1: nothing to
// prefetch) with the CTA's first loads, and future_tile_prefetch, called
// once the prologue is done (the load has long returned), asks L2 for the
// tile.
struct FutureTile {
  int s, h, tile;
};
// (self, n_units): the calling CTA's work unit and the launch's number of
// units (a CTA per unit: blockIdx.x and gridDim.x, the defaults).
__device__ __forceinline__ FutureTile future_tile_begin(const StepParams& p, int self,
                                                        int n_units) {
  FutureTile f{-1, 0, 0};
  const long long fut = (long long)self + p.prefetch_ahead;
  if (p.prefetch_ahead <= 0 || fut >= (long long)n_units) return f;
  const int fi = (int)fut;
  const int bh = fdiv(fi, p.div_tiles);
  f.tile = fi - bh * (int)p.div_tiles.d;
  const int b = fdiv(bh, p.div_h);
  f.h = bh - b * p.H;
  f.s = __ldg(p.slot_idx + b);
  return f;
}
__device__ __forceinline__ FutureTile future_tile_begin(const StepParams& p) {
  return future_tile_begin(p, (int)blockIdx.x, (int)gridDim.x);
}
template <typename StT>
__device__ __forceinline__ void future_tile_prefetch(const StepParams& p, const FutureTile& f,
                                                     int rows_cta, int dk) {
  if (f.s < 0 || (p.n_slots > 0 && f.s >= p.n_slots)) return;
  const StT* src = reinterpret_cast<const StT*>(p.state) +
                   (((size_t)f.s * p.H + f.h) * p.dv + (size_t)f.tile * rows_cta) * dk;
  prefetch_l2(src, (unsigned)(rows_cta * dk * sizeof(StT)));
}

// The same CTA's per-token inputs, one lane per request (lanes 0 .. 4T-1 of
// the calling warp, T <= 8): q and k of each token (dk values each), the v
// values of the tile's rows, and the lines holding each token's gate and
// beta.  Called by a whole warp; (self, n_units) as for future_tile_begin.
template <typename InT>
__device__ __forceinline__ void prefetch_future_inputs(const StepParams& p, int rows_cta, int dk,
                                                       int lane, int self, int n_units) {
  const long long fut = (long long)self + p.prefetch_ahead;
  if (p.prefetch_ahead <= 0 || fut >= (long long)n_units || lane >= 4 * p.T) return;
  const int f = (int)fut;
  const int bh = fdiv(f, p.div_tiles), tile = f - bh * (int)p.div_tiles.d;
  const int b = fdiv(bh, p.div_h), h = bh - b * p.H;
  if (lane >= 3 * p.T) {
    const size_t bth = ((size_t)b * p.T + (lane - 3 * p.T)) * p.H + h;
    prefetch_l2_line(p.g + bth);
    prefetch_l2_line(p.beta + bth);
    return;
  }
  const int t = lane / 3, which = lane % 3;
  const size_t bt = (size_t)b * p.T + t;
  if (which < 2) {
    const InT* src = reinterpret_cast<const InT*>(which == 0 ? p.q : p.k) +
                     (bt * p.Hk + fdiv(h, p.div_group)) * dk;
    prefetch_l2(src, (unsigned)(dk * sizeof(InT)));
  } else {
    const InT* src = reinterpret_cast<const InT*>(p.v) + (bt * p.H + h) * p.dv +
                     (size_t)tile * rows_cta;
    prefetch_l2(src, (unsigned)(rows_cta * sizeof(InT)));
  }
}
template <typename InT>
__device__ __forceinline__ void prefetch_future_inputs(const StepParams& p, int rows_cta, int dk,
                                                       int lane) {
  prefetch_future_inputs<InT>(p, rows_cta, dk, lane, (int)blockIdx.x, (int)gridDim.x);
}

// Grid: one CTA per (b, h, tile of W * 32/LPR * M rows); block: W warps.
// Block index order is tile fastest, then h, then b, so consecutive CTAs
// stream consecutive state memory of a slot.  Dynamic shared memory holds
// the call's normalised q and k: T * (2 * DK + 1) floats, written once per
// CTA by its warps (token t by warp t % W) before the rows are updated.
// ONE (single-token calls): every warp normalises the token's q and k into a
// copy of its own, W * (2 * DK + 4) floats, so no warp waits at a CTA barrier
// for another's prologue (same arithmetic, same bits).
// PACKED (16-bit states, single-token calls only) keeps the rows packed in
// registers, so a warp holds twice the rows for the same registers.
template <int DK, int LPR, int M, int W, typename InT, typename OutT, typename StT, bool PACKED,
          bool ONE>
__global__ void __launch_bounds__(W * 32) decode_kernel(const StepParams p) {
  constexpr int CW = StateTraits<StT>::CW;
  using L = Lanes<DK, LPR, CW>;
  constexpr int EL = L::EL;
  constexpr int ROWS_W = L::GROUPS * M;
  constexpr int ROWS_CTA = W * ROWS_W;
  static_assert(!PACKED || sizeof(StT) == 2, "only 16-bit rows are kept packed");
  static_assert(!PACKED || ONE, "packed rows are for single-token calls");
  extern __shared__ __align__(16) float dq_smem[];  // [T][2][DK], then [T] k.q; ONE: per warp
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  float* qk_smem = ONE ? dq_smem + (size_t)warp * (2 * DK + 4) : dq_smem;
  const int pos = lane % LPR;
  const int bh = fdiv((int)blockIdx.x, p.div_tiles);
  const int tile = (int)blockIdx.x - bh * (int)p.div_tiles.d;
  const int b = fdiv(bh, p.div_h), h = bh - b * p.H;
  const int j0 = tile * ROWS_CTA + warp * ROWS_W + (lane / LPR) * M;  // this group's rows
  const int kh = fdiv(h, p.div_group);
  OutT* out = reinterpret_cast<OutT*>(p.out);

  // one slot per CTA: every warp of the CTA takes the same branch
  const int s = __ldg(p.slot_idx + b);
  if (s < 0 || (p.n_slots > 0 && s >= p.n_slots)) {
    if (s != -1 && p.dev_status != nullptr && lane == 0)
      atomicOr(p.dev_status, GDN_STATUS_SLOT_RANGE);
    if (pos < M) {
      for (int t = 0; t < p.T; ++t)
        store_scalar(out + (((size_t)b * p.T + t) * p.H + h) * p.dv + j0 + pos, 0.0f);
    }
    return;
  }

  // where the state goes: after the last token into slot s (default); after
  // token n_accept[b] - 1 into slot s (commit); after every token t into
  // token_slots[b][t] (snapshots)
  int n_commit = p.T;
  if (p.n_accept != nullptr) {
    n_commit = __ldg(p.n_accept + b);
    if (n_commit < 0 || n_commit > p.T) {
      if (p.dev_status != nullptr && lane == 0) atomicOr(p.dev_status, GDN_STATUS_ACCEPT_RANGE);
      n_commit = 0;
    }
  }
  const size_t slot_stride = (size_t)p.H * p.dv * DK;
  const size_t row_off = ((size_t)h * p.dv + j0) * DK + pos * CW;

  // the state rows are requested first, so they are in flight while q and k
  // are normalised
  StT* sp = reinterpret_cast<StT*>(p.state) + (((size_t)s * p.H + h) * p.dv + j0) * DK;
  StT* lane_sp = sp + pos * CW;  // every row and chunk is a constant offset from here
  float S[PACKED ? 1 : M][PACKED ? 1 : EL];
  uint32_t P[PACKED ? M : 1][PACKED ? EL / 2 : 1];
#pragma unroll
  for (int m = 0; m < M; ++m) {
    if constexpr (PACKED) {
#pragma unroll
      for (int c = 0; c < L::CH; ++c) {
        const uint4 t = __ldcs(reinterpret_cast<const uint4*>(lane_sp + m * DK + c * LPR * CW));
        P[m][4 * c + 0] = t.x;
        P[m][4 * c + 1] = t.y;
        P[m][4 * c + 2] = t.z;
        P[m][4 * c + 3] = t.w;
      }
    } else {
      load_row<StT, DK, LPR>(sp + (size_t)m * DK, pos, S[m]);
    }
  }

  if (threadIdx.x == (W - 1) * 32)
    future_tile_prefetch<StT>(p, future_tile_begin(p), ROWS_CTA, DK);

  // every token's v values of the tile's rows and its gates are requested
  // now, so that their latencies overlap those of the state and of q and k:
  // one token's into registers, several tokens' into shared memory for the
  // token loop
  constexpr int kMaxT = 8;
  constexpr int VT = ONE ? 1 : kMaxT, VR = ONE ? 1 : ROWS_CTA;
  constexpr int VPT = ONE ? 1 : (kMaxT * ROWS_CTA + W * 32 - 1) / (W * 32);  // v values per thread
  __shared__ float v_s[VT][VR];
  __shared__ float tok_s[2][VT];
  float v_pre[VPT], g_pre = 0.0f, b_pre = 0.0f;
  float v_one[ONE ? M : 1];  // one token: this group's v values, requested now too
  if (warp == W - 1) prefetch_future_inputs<InT>(p, ROWS_CTA, DK, lane);
  if constexpr (ONE) {
    load_vec<InT, M>(reinterpret_cast<const InT*>(p.v) + ((size_t)b * p.H + h) * p.dv + j0, v_one);
    g_pre = __ldg(p.g + (size_t)b * p.H + h);
    b_pre = __ldg(p.beta + (size_t)b * p.H + h);
  } else {
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int i = threadIdx.x + k * W * 32;
      if (i < p.T * ROWS_CTA) {
        const int t = i / ROWS_CTA, r = i % ROWS_CTA;
        float v1[1];
        load_vec<InT, 1>(reinterpret_cast<const InT*>(p.v) +
                             (((size_t)b * p.T + t) * p.H + h) * p.dv + tile * ROWS_CTA + r,
                         v1);
        v_pre[k] = v1[0];
      }
    }
    if (threadIdx.x < p.T) {
      const size_t bth = ((size_t)b * p.T + threadIdx.x) * p.H + h;
      g_pre = __ldg(p.g + bth);
      b_pre = __ldg(p.beta + bth);
    }
  }

  float* kq_s = qk_smem + (size_t)p.T * 2 * DK;
  if constexpr (ONE) {
    const size_t base = ((size_t)b * p.Hk + kh) * DK;
    normalise_qk<InT, DK>(reinterpret_cast<const InT*>(p.k) + base,
                          reinterpret_cast<const InT*>(p.q) + base, lane, p.l2_eps, p.l2norm,
                          qk_smem, qk_smem + DK, kq_s);
    __syncwarp();
  } else {
    for (int t = warp; t < p.T; t += W) {
      const size_t base = (((size_t)b * p.T + t) * p.Hk + kh) * DK;
      normalise_qk<InT, DK>(reinterpret_cast<const InT*>(p.k) + base,
                            reinterpret_cast<const InT*>(p.q) + base, lane, p.l2_eps, p.l2norm,
                            qk_smem + (size_t)t * 2 * DK, qk_smem + (size_t)t * 2 * DK + DK,
                            kq_s + t);
    }
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int i = threadIdx.x + k * W * 32;
      if (i < p.T * ROWS_CTA) v_s[i / ROWS_CTA][i % ROWS_CTA] = v_pre[k];
    }
    if (threadIdx.x < p.T) {
      tok_s[0][threadIdx.x] = expf(g_pre);
      tok_s[1][threadIdx.x] = b_pre;
    }
    __syncthreads();
  }

  // store this lane's rows into pool slot `slot`
  auto store_rows = [&](int slot) {
    StT* dst = reinterpret_cast<StT*>(p.state) + (size_t)slot * slot_stride + row_off;
#pragma unroll
    for (int m = 0; m < M; ++m) {
      if constexpr (PACKED) {
#pragma unroll
        for (int c = 0; c < L::CH; ++c)
          __stcs(reinterpret_cast<uint4*>(dst + m * DK + c * LPR * CW),
                 make_uint4(P[m][4 * c + 0], P[m][4 * c + 1], P[m][4 * c + 2], P[m][4 * c + 3]));
      } else {
        store_row<StT, DK, LPR>(dst - pos * CW + (size_t)m * DK, pos, S[m]);
      }
    }
  };

  TokenScalars ts;
  ts.scale = p.scale;
  const int T = PACKED ? 1 : p.T;  // packed rows: single-token calls only
  for (int t = 0; t < T; ++t) {
    const size_t bt = (size_t)b * p.T + t;
    float vv[M];
    if constexpr (ONE) {
#pragma unroll
      for (int m = 0; m < M; ++m) vv[m] = v_one[m];
      ts.alpha = expf(g_pre);
      ts.beta = b_pre;
    } else {
      const int jl = j0 - tile * ROWS_CTA;
#pragma unroll
      for (int m = 0; m < M; ++m) vv[m] = v_s[t][jl + m];
      ts.alpha = tok_s[0][t];
      ts.beta = tok_s[1][t];
    }
    ts.kq = kq_s[t];
    float o[M];
    if constexpr (PACKED) {
      token_rows_packed<StT, DK, LPR, M>(P, qk_smem + (size_t)t * 2 * DK,
                                         qk_smem + (size_t)t * 2 * DK + DK, pos, vv, ts, o);
    } else {
      float kn[EL], qn[EL];
      lanes_from_smem<DK, LPR, CW>(qk_smem + (size_t)t * 2 * DK, pos, kn);
      lanes_from_smem<DK, LPR, CW>(qk_smem + (size_t)t * 2 * DK + DK, pos, qn);
      token_rows<LPR, EL, M>(S, kn, qn, vv, ts, o);
    }
    const float mine = select_row<M>(o, pos);
    if (pos < M) store_scalar(out + (bt * p.H + h) * p.dv + j0 + pos, mine);
    if (p.token_slots != nullptr) {
      const int ts_slot = __ldg(p.token_slots + bt);
      if (ts_slot >= 0 && (p.n_slots <= 0 || ts_slot < p.n_slots)) {
        store_rows(ts_slot);
      } else if (ts_slot != -1 && p.dev_status != nullptr && lane == 0) {
        atomicOr(p.dev_status, GDN_STATUS_SLOT_RANGE);
      }
    } else if (t + 1 == n_commit) {
      store_rows(s);
    }
  }
}

// ---------------------------------------------------------------------------
// up to four tokens at once: the block form of the recurrence
//
// Unrolling the gated delta rule over the tokens of one call writes every
// quantity of token t in terms of the state S0 the call starts from.  With
// a_t = exp(g_t), D_t = a_0 a_1 ... a_t and G(s, t) = a_{s+1} ... a_t (G(t, t)
// = 1), for every row j of the state (one dv index):
//   p_t = D_t (S0_j . k_t) + sum_{s<t} G(s, t) (k_s . k_t) d_s      (prediction)
//   d_t = beta_t (v_tj - p_t)
//   o_tj = scale (D_t (S0_j . q_t) + sum_{s<t} G(s, t) (k_s . q_t) d_s + (k_t . q_t) d_t)
//   S_n,j = D_{n-1} S0_j + sum_{s<n} G(s, n-1) d_s k_s            (after n tokens)
// So one pass over the rows takes all 2T dot products with S0, one
// reduction over the lane group serves every token, the token-to-token
// dependence is a short scalar recurrence, and each stored state is one
// rank-n update of S0 (1 + n operations per element instead of 2n).  For
// n = 1 every expression is the single-token one, operation for operation,
// so with the same lane partition the first token's output and state carry
// the same bits as a single-token call.

// Reduce-scatter N values over each aligned group of LPR lanes: after it the
// lane at group position pos holds the complete sums of values
// [pos*N/LPR, (pos+1)*N/LPR) in x[0 .. N/LPR).  Levels run from the widest
// offset down, as in group_allreduce, and every partial sum adds the same two
// operands as there, so each sum has the bits the all-reduce gives.
template <int LPR, int N>
__device__ __forceinline__ void group_reduce_scatter(float (&x)[N], int pos) {
  static_assert(N % LPR == 0, "whole values per lane");
  int n = N;
#pragma unroll
  for (int off = LPR / 2; off >= 1; off >>= 1) {
    n >>= 1;
    const bool upper = (pos & off) != 0;
#pragma unroll
    for (int i = 0; i < n; ++i) {
      const float send = upper ? x[i] : x[i + n];
      const float keep = upper ? x[i + n] : x[i];
      x[i] = __fadd_rn(keep, __shfl_xor_sync(kFull, send, off));
    }
  }
}

constexpr int kBlockTokens = 4;  // longest call taken in block form

// ---------------------------------------------------------------------------
// bulk copies into shared memory, completed on an mbarrier (no multicast)

__device__ __forceinline__ uint32_t smem_u32(const void* ptr) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Orders this thread's generic shared-memory accesses before later
// async-proxy ones (a bulk copy into the same bytes).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// One bulk copy of `bytes` (a multiple of 16; both addresses 16-byte
// aligned) from global memory into this CTA's shared memory.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, unsigned bytes,
                                              uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
  return t;
}

// Wait for an mbarrier phase, giving up after `limit_ns` nanoseconds.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity,
                                                  uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
}

// a copy that has not landed after a second never will
#ifndef GDN_WAIT_LIMIT_NS
#define GDN_WAIT_LIMIT_NS 1000000000ull
#endif
constexpr uint64_t kWaitLimitNs = GDN_WAIT_LIMIT_NS;

// Test builds of the library only (the shipped build leaves it at 0):
// transaction bytes that the bulk-copy waits of the multi-token block forms
// (CUDA cores and tensor cores), of the staged 16-bit single-token kernel
// and of the low-rank kernel expect on top of what their copy delivers.  A
// copy of N bytes against an expectation of N + extra never completes the
// mbarrier phase, although every byte lands: the wait runs out at its limit
// without any fault, which is how a test drives the timeout branch.
#ifndef GDN_WAIT_TEST_EXTRA_TX
#define GDN_WAIT_TEST_EXTRA_TX 0u
#endif
constexpr unsigned kWaitTestExtraTx = GDN_WAIT_TEST_EXTRA_TX;

// ---------------------------------------------------------------------------
// the block form, with the state tile in shared memory
//
// The CTA's state tile is brought into shared memory by one bulk copy and
// read from there twice (the dot products, then the update on its way back
// to HBM), so no registers hold it: 5 CTAs fit on an SM instead of the 4 a
// register-resident tile allows, and each keeps its whole tile in flight at
// no register cost.

// 4 consecutive state elements from shared memory, widened to fp32.
template <typename St>
__device__ __forceinline__ void lds4(const St* p, float (&x)[4]) {
  if constexpr (sizeof(St) == 4) {
    const float4 t = *reinterpret_cast<const float4*>(p);
    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
  } else {
    const uint2 t = *reinterpret_cast<const uint2*>(p);
    unpack2(St(), t.x, x[0], x[1]);
    unpack2(St(), t.y, x[2], x[3]);
  }
}

// Rows of the state after n tokens, S_n = D_{n-1} S0 + sum_{u<n} G(u, n-1)
// d_u k_u, from the shared-memory tile rows Ss_row (this lane's group's
// first row) into dst, 4 elements at a time.  al holds the call's decays
// a_t, dm[m][u] row m's d_u, kn_s the normalised k of token u at kn_s + u *
// 2 * DK.  N is a compile-time bound on n (n = N unless passed): the same
// operations run for every n <= N, those of tokens u >= n skipped, and D and
// G are formed left to right as in the kernel.
template <int N, int TT, int DK, int LPR, int M, typename StT>
__device__ __forceinline__ void store_block_state_smem(StT* dst, const StT* Ss_row,
                                                       const float* kn_s, int pos,
                                                       const float (&al)[TT],
                                                       const float (&dm)[M][TT], int n = N) {
  constexpr int CW = StateTraits<StT>::CW;
  using L = Lanes<DK, LPR, CW>;
  float Dn = al[0], Gn[N];
#pragma unroll
  for (int t = 1; t < N; ++t)
    if (t < n) Dn = __fmul_rn(Dn, al[t]);
#pragma unroll
  for (int u = 0; u < N; ++u) {
    Gn[u] = 1.0f;
#pragma unroll
    for (int t = u + 1; t < N; ++t)
      if (t < n) Gn[u] = __fmul_rn(Gn[u], al[t]);
  }
  float cf[M][N];
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int u = 0; u < N; ++u) cf[m][u] = __fmul_rn(Gn[u], dm[m][u]);
  // 4 elements at a time (a whole fp32 chunk, half a 16-bit one)
#pragma unroll
  for (int c = 0; c < L::CH; ++c) {
#pragma unroll
    for (int i0 = 0; i0 < CW; i0 += 4) {
      float kc[N][4];
#pragma unroll
      for (int u = 0; u < N; ++u) {
        if (u < n) {
          const float4 k4 = *reinterpret_cast<const float4*>(kn_s + (size_t)u * 2 * DK +
                                                             L::offset(pos, c) + i0);
          kc[u][0] = k4.x; kc[u][1] = k4.y; kc[u][2] = k4.z; kc[u][3] = k4.w;
        }
      }
#pragma unroll
      for (int m = 0; m < M; ++m) {
        float x[4], y[4];
        lds4<StT>(Ss_row + (size_t)m * DK + L::offset(pos, c) + i0, x);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          y[i] = __fmul_rn(Dn, x[i]);
#pragma unroll
          for (int u = 0; u < N; ++u)
            if (u < n) y[i] = __fmaf_rn(kc[u][i], cf[m][u], y[i]);
        }
        StT* q = dst + (size_t)m * DK + L::offset(pos, c) + i0;
        if constexpr (sizeof(StT) == 4) {
          __stcs(reinterpret_cast<float4*>(q), make_float4(y[0], y[1], y[2], y[3]));
        } else {
          __stcs(reinterpret_cast<uint2*>(q),
                 make_uint2(pack2(StT(), y[0], y[1]), pack2(StT(), y[2], y[3])));
        }
      }
    }
  }
}

// Dynamic shared memory: the tile (ROWS_CTA x DK of StT, 16-byte aligned),
// then the call's normalised q and k ([TT][2][DK]) and the k.q values.
template <int TT, int DK, int ROWS_CTA, typename StT>
__host__ __device__ constexpr size_t block_smem_bytes() {
  return (size_t)ROWS_CTA * DK * sizeof(StT) + (size_t)TT * (2 * DK + 1) * sizeof(float);
}

// Dot products of the group's M tile rows with the normalised k and q of
// tokens T0 .. T0+NT-1, reduce-scattered over the group: afterwards lane
// 2m (2m + 1) of the group holds row m's S0.k_t (S0.q_t) in X[T0 + t].  Each
// sum runs over the row's elements in increasing order and takes the same
// butterfly whatever the token range, so splitting the tokens over several
// calls changes no bits.
template <int T0, int NT, int TT, int DK, int LPR, int M, typename StT>
__device__ __forceinline__ void block_dots(const StT* Ss_row, const float* qk_smem, int pos,
                                           float (&X)[TT]) {
  constexpr int CW = StateTraits<StT>::CW;
  using L = Lanes<DK, LPR, CW>;
  if constexpr (2 * M == LPR && (NT & (NT - 1)) == 0) {
    // Without selects: the reduce-scatter's value v = (m * 2 + kq) * NT + t
    // is accumulated by lane pos in register r = v ^ (NT * pos), i.e. register
    // group g holds (m * 2 + kq) = g ^ pos.  Then at every level each lane
    // keeps its lower half of registers and sends the upper half, whose
    // values are exactly the partner's lower half: the same sums, added in
    // the same order, as group_reduce_scatter, with no per-lane selects.  The
    // row of group pair j (j ^ (pos / 2)) and the k / q operand of group
    // 2j + b (b ^ (pos & 1)) become per-lane shared-memory addresses.
    float acc[2 * M][NT];
    const int pp = pos >> 1;
    const StT* rows[M];
#pragma unroll
    for (int j = 0; j < M; ++j) rows[j] = Ss_row + (size_t)(j ^ pp) * DK + L::offset(pos, 0);
    const float* op0 = qk_smem + (pos & 1) * DK + L::offset(pos, 0);
    const float* op1 = qk_smem + ((pos & 1) ^ 1) * DK + L::offset(pos, 0);
#pragma unroll
    for (int c = 0; c < L::CH; ++c) {
#pragma unroll
      for (int i0 = 0; i0 < CW; i0 += 4) {
        const int co = CW * LPR * c + i0;  // L::offset(pos, c) - L::offset(pos, 0)
        float a0[NT][4], a1[NT][4];
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const float4 u0 = *reinterpret_cast<const float4*>(op0 + (T0 + t) * 2 * DK + co);
          const float4 u1 = *reinterpret_cast<const float4*>(op1 + (T0 + t) * 2 * DK + co);
          a0[t][0] = u0.x; a0[t][1] = u0.y; a0[t][2] = u0.z; a0[t][3] = u0.w;
          a1[t][0] = u1.x; a1[t][1] = u1.y; a1[t][2] = u1.z; a1[t][3] = u1.w;
        }
#pragma unroll
        for (int j = 0; j < M; ++j) {
          float x[4];
          lds4<StT>(rows[j] + co, x);
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            float& r0 = acc[2 * j][t];
            float& r1 = acc[2 * j + 1][t];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              if (c == 0 && i0 == 0 && i == 0) {
                r0 = __fmul_rn(x[0], a0[t][0]);
                r1 = __fmul_rn(x[0], a1[t][0]);
              } else {
                r0 = __fmaf_rn(x[i], a0[t][i], r0);
                r1 = __fmaf_rn(x[i], a1[t][i], r1);
              }
            }
          }
        }
      }
    }
    float red[2 * M * NT];
#pragma unroll
    for (int g = 0; g < 2 * M; ++g)
#pragma unroll
      for (int t = 0; t < NT; ++t) red[g * NT + t] = acc[g][t];
    int n = 2 * M * NT;
#pragma unroll
    for (int off = LPR / 2; off >= 1; off >>= 1) {
      n >>= 1;
#pragma unroll
      for (int i = 0; i < n; ++i) red[i] = __fadd_rn(red[i], __shfl_xor_sync(kFull, red[i + n], off));
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) X[T0 + t] = red[t];
    return;
  }
  float red[2 * M * NT];  // [(m * 2 + k or q) * NT + t]
#pragma unroll
  for (int c = 0; c < L::CH; ++c) {
#pragma unroll
    for (int i0 = 0; i0 < CW; i0 += 4) {
      float kc[NT][4], qc[NT][4];
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const float* kn = qk_smem + (T0 + t) * 2 * DK + L::offset(pos, c) + i0;
        const float4 k4 = *reinterpret_cast<const float4*>(kn);
        const float4 q4 = *reinterpret_cast<const float4*>(kn + DK);
        kc[t][0] = k4.x; kc[t][1] = k4.y; kc[t][2] = k4.z; kc[t][3] = k4.w;
        qc[t][0] = q4.x; qc[t][1] = q4.y; qc[t][2] = q4.z; qc[t][3] = q4.w;
      }
#pragma unroll
      for (int m = 0; m < M; ++m) {
        float x[4];
        lds4<StT>(Ss_row + (size_t)m * DK + L::offset(pos, c) + i0, x);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          float& rk = red[(m * 2 + 0) * NT + t];
          float& rq = red[(m * 2 + 1) * NT + t];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (c == 0 && i0 == 0 && i == 0) {
              rk = __fmul_rn(x[0], kc[t][0]);
              rq = __fmul_rn(x[0], qc[t][0]);
            } else {
              rk = __fmaf_rn(x[i], kc[t][i], rk);
              rq = __fmaf_rn(x[i], qc[t][i], rq);
            }
          }
        }
      }
    }
  }
  group_reduce_scatter<LPR, 2 * M * NT>(red, pos);
#pragma unroll
  for (int t = 0; t < NT; ++t) X[T0 + t] = red[t];
}

// Grid and block as decode_kernel; calls of exactly TT tokens (2..4).  M =
// LPR / 2 rows per group, so after the reduce-scatter of the 2 * M * TT
// sums, lane 2m of a group holds row m's S0.k_t (t < TT) and lane 2m + 1 its
// S0.q_t.  The per-token scalars, the tile's v and the Gram entries k_u.k_t
// and k_u.q_t (u < t) are staged in static shared memory.  SPEC: the call
// carries n_accept or token_slots (the state after fewer tokens, or after
// every token, is stored); otherwise the state after all TT tokens goes back
// to its slot, with no other store path compiled in.  96 registers at 5
// CTAs per SM (the tile's 32 KB x 5 fits the SM's shared memory).
template <int TT, int DK, int LPR, int W, typename InT, typename OutT, typename StT, bool SPEC>
__global__ void __launch_bounds__(W * 32, 5) decode_block_smem_kernel(const StepParams p) {
  static_assert(TT >= 2 && TT <= kBlockTokens, "block calls take 2..4 tokens");
  constexpr int M = LPR / 2;
  constexpr int CW = StateTraits<StT>::CW;
  using L = Lanes<DK, LPR, CW>;
  constexpr int ROWS_CTA = W * L::GROUPS * M;
  constexpr int E32 = DK / 32;
  constexpr int NPAIR = TT * (TT - 1) / 2;
  constexpr unsigned TILE_BYTES = ROWS_CTA * DK * sizeof(StT);
  extern __shared__ __align__(128) unsigned char blk_smem[];
  StT* Ss = reinterpret_cast<StT*>(blk_smem);                         // [ROWS_CTA][DK]
  float* qk_smem = reinterpret_cast<float*>(blk_smem + TILE_BYTES);   // [TT][2][DK], [TT]
  __shared__ float gram[2][NPAIR];
  __shared__ float tok_s[2][TT];
  __shared__ float v_s[TT][ROWS_CTA];
  __shared__ uint64_t bar;
  __shared__ int landed;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int pos = lane % LPR;
  const int bh = fdiv((int)blockIdx.x, p.div_tiles);
  const int tile = (int)blockIdx.x - bh * (int)p.div_tiles.d;
  const int b = fdiv(bh, p.div_h), h = bh - b * p.H;
  const int row0 = tile * ROWS_CTA;
  const int jl = warp * L::GROUPS * M + (lane / LPR) * M;  // this group's first row in the tile
  const int j0 = row0 + jl;
  const int kh = fdiv(h, p.div_group);
  OutT* out = reinterpret_cast<OutT*>(p.out);

  // The per-token inputs are requested before the slot, which none of them
  // depends on, in the order their results are needed: token `warp`'s k and
  // q (one token per warp: straight into registers), the tile's v values and
  // the gates (into shared memory after the first barrier).  The slot of the
  // CTA prefetch_ahead on is requested too, for the L2 prefetch of its tile.
  constexpr bool QK_REG = TT <= W;
  float kv[E32], qv[E32];
  if constexpr (QK_REG) {
    if (warp < TT) {
      const size_t base = (((size_t)b * TT + warp) * p.Hk + kh) * DK;
      load_vec<InT, E32>(reinterpret_cast<const InT*>(p.k) + base + lane * E32, kv);
      load_vec<InT, E32>(reinterpret_cast<const InT*>(p.q) + base + lane * E32, qv);
    }
  }
  constexpr int VPT = (TT * ROWS_CTA + W * 32 - 1) / (W * 32);  // v values per thread
  float v_pre[VPT], g_pre = 0.0f, b_pre = 0.0f;
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    const int i = threadIdx.x + k * W * 32;
    if (i < TT * ROWS_CTA) {
      const int t = i / ROWS_CTA, r = i % ROWS_CTA;
      float v1[1];
      load_vec<InT, 1>(reinterpret_cast<const InT*>(p.v) +
                           (((size_t)b * TT + t) * p.H + h) * p.dv + row0 + r, v1);
      v_pre[k] = v1[0];
    }
  }
  if (threadIdx.x < TT) {
    const size_t bth = ((size_t)b * TT + threadIdx.x) * p.H + h;
    g_pre = __ldg(p.g + bth);
    b_pre = __ldg(p.beta + bth);
  }
  FutureTile fut{-1, 0, 0};
  if (threadIdx.x == (W - 1) * 32) fut = future_tile_begin(p);

  const int s = __ldg(p.slot_idx + b);
  if (s < 0 || (p.n_slots > 0 && s >= p.n_slots)) {
    if (s != -1 && p.dev_status != nullptr && lane == 0)
      atomicOr(p.dev_status, GDN_STATUS_SLOT_RANGE);
    if (pos < M) {
#pragma unroll
      for (int t = 0; t < TT; ++t)
        store_scalar(out + (((size_t)b * TT + t) * p.H + h) * p.dv + j0 + pos, 0.0f);
    }
    return;
  }
  int n_commit = TT;
  if (SPEC && p.n_accept != nullptr) {
    n_commit = __ldg(p.n_accept + b);
    if (n_commit < 0 || n_commit > TT) {
      if (p.dev_status != nullptr && lane == 0) atomicOr(p.dev_status, GDN_STATUS_ACCEPT_RANGE);
      n_commit = 0;
    }
  }

  // the tile: one bulk copy, completed on the mbarrier
  const StT* src = reinterpret_cast<const StT*>(p.state) + (((size_t)s * p.H + h) * p.dv + row0) * DK;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&bar, TILE_BYTES + kWaitTestExtraTx);
    bulk_copy_g2s(Ss, src, TILE_BYTES, &bar);
  }
  const int mr = pos >> 1;
  const bool is_q = (pos & 1) != 0;

  float* kq_s = qk_smem + TT * 2 * DK;
  if constexpr (QK_REG) {
    if (warp < TT)
      normalise_loaded<DK>(kv, qv, lane, p.l2_eps, p.l2norm, qk_smem + warp * 2 * DK,
                           qk_smem + warp * 2 * DK + DK, kq_s + warp);
  } else {
    for (int t = warp; t < TT; t += W) {
      const size_t base = (((size_t)b * TT + t) * p.Hk + kh) * DK;
      normalise_qk<InT, DK>(reinterpret_cast<const InT*>(p.k) + base,
                            reinterpret_cast<const InT*>(p.q) + base, lane, p.l2_eps, p.l2norm,
                            qk_smem + t * 2 * DK, qk_smem + t * 2 * DK + DK, kq_s + t);
    }
  }
  __syncthreads();
  // the L2 prefetches for the CTA prefetch_ahead on, off the prologue's path
  if (threadIdx.x == (W - 1) * 32) future_tile_prefetch<StT>(p, fut, ROWS_CTA, DK);
  if (warp == W - 1) prefetch_future_inputs<InT>(p, ROWS_CTA, DK, lane);
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    const int i = threadIdx.x + k * W * 32;
    if (i < TT * ROWS_CTA) v_s[i / ROWS_CTA][i % ROWS_CTA] = v_pre[k];
  }
  if (threadIdx.x < TT) {
    tok_s[0][threadIdx.x] = expf(g_pre);
    tok_s[1][threadIdx.x] = b_pre;
  }
  for (int i = warp; i < 2 * NPAIR; i += W) {
    const int which = i / NPAIR, pr = i % NPAIR;
    int t = 1;
    while (pr >= t * (t + 1) / 2) ++t;
    const int u = pr - t * (t - 1) / 2;
    float x[E32], y[E32];
    load_vec<float, E32>(qk_smem + u * 2 * DK + lane * E32, x);
    load_vec<float, E32>(qk_smem + t * 2 * DK + which * DK + lane * E32, y);
    float acc[1];
    acc[0] = __fmul_rn(x[0], y[0]);
#pragma unroll
    for (int e = 1; e < E32; ++e) acc[0] = __fmaf_rn(x[e], y[e], acc[0]);
    group_allreduce<32, 1>(acc);
    if (lane == 0) gram[which][pr] = acc[0];
  }
  if (threadIdx.x == 0) landed = mbar_wait_bounded(&bar, 0, kWaitLimitNs) ? 1 : 0;
  __syncthreads();
  if (!landed) {
    // the copy did not land: report it, give it one more bounded wait so the
    // shared memory is not released under it, and leave the state as it was
    if (threadIdx.x == 0) {
      if (p.dev_status != nullptr) atomicOr(p.dev_status, GDN_STATUS_TIMEOUT);
      mbar_wait_bounded(&bar, 0, kWaitLimitNs);
    }
    return;
  }
  mbar_try_wait(&bar, 0);  // completed: every thread acquires the copied bytes

  // all 2 * TT dot products of every row with S0, from the tile
  const StT* Ss_row = Ss + (size_t)jl * DK;
  float red[TT];  // S0_mr . k_t (even pos) or S0_mr . q_t (odd pos)
  block_dots<0, TT, TT, DK, LPR, M, StT>(Ss_row, qk_smem, pos, red);

  float al[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) al[t] = tok_s[0][t];
  float D[TT], G[TT][TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) D[t] = t == 0 ? al[0] : __fmul_rn(D[t - 1], al[t]);
#pragma unroll
  for (int u = 0; u < TT; ++u) {
    G[u][u] = 1.0f;
#pragma unroll
    for (int t = u + 1; t < TT; ++t) G[u][t] = __fmul_rn(G[u][t - 1], al[t]);
  }
  float dd[TT];
  const int pair = lane & ~1;
  const float* gram_mine = gram[is_q ? 1 : 0];
#pragma unroll
  for (int t = 0; t < TT; ++t) {
    float x = __fmul_rn(D[t], red[t]);
#pragma unroll
    for (int u = 0; u < t; ++u)
      x = __fmaf_rn(__fmul_rn(G[u][t], gram_mine[t * (t - 1) / 2 + u]), dd[u], x);
    const float dt = __fmul_rn(tok_s[1][t], __fsub_rn(v_s[t][jl + mr], x));
    dd[t] = __shfl_sync(kFull, dt, pair);
    if (is_q) {
      const float o = __fmul_rn(p.scale, __fmaf_rn(kq_s[t], dd[t], x));
      store_scalar(out + (((size_t)b * TT + t) * p.H + h) * p.dv + j0 + mr, o);
    }
  }
  float dm[M][TT];
  const int gbase = lane & ~(LPR - 1);
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int t = 0; t < TT; ++t) dm[m][t] = __shfl_sync(kFull, dd[t], gbase + 2 * m);

  const size_t slot_stride = (size_t)p.H * p.dv * DK;
  const size_t row_off = ((size_t)h * p.dv + j0) * DK;
  if (!SPEC) {
    store_block_state_smem<TT, TT, DK, LPR, M, StT>(
        reinterpret_cast<StT*>(p.state) + (size_t)s * slot_stride + row_off, Ss_row, qk_smem, pos,
        al, dm);
  } else if (p.token_slots != nullptr) {
#pragma unroll 1
    for (int t = 0; t < TT; ++t) {
      const int ts_slot = __ldg(p.token_slots + (size_t)b * TT + t);
      if (ts_slot >= 0 && (p.n_slots <= 0 || ts_slot < p.n_slots)) {
        store_block_state_smem<TT, TT, DK, LPR, M, StT>(
            reinterpret_cast<StT*>(p.state) + (size_t)ts_slot * slot_stride + row_off, Ss_row,
            qk_smem, pos, al, dm, t + 1);
      } else if (ts_slot != -1 && p.dev_status != nullptr && lane == 0) {
        atomicOr(p.dev_status, GDN_STATUS_SLOT_RANGE);
      }
    }
  } else if (n_commit > 0) {
    store_block_state_smem<TT, TT, DK, LPR, M, StT>(
        reinterpret_cast<StT*>(p.state) + (size_t)s * slot_stride + row_off, Ss_row, qk_smem, pos,
        al, dm, n_commit);
  }
}

// ---------------------------------------------------------------------------
// single-token calls on a 16-bit pool, with the tile staged in shared memory
//
// The packed kernel (decode_kernel with PACKED) holds its rows in registers
// from the load to the store, so the bytes an SM keeps in flight are bounded
// by its registers (8 CTAs of 8 KB at 118 registers per thread).  Here one
// bulk copy brings a CTA's 64-row tile into shared memory and each lane reads
// its rows from there twice (the dot products, then the update on its way
// back to HBM), so bytes in flight cost no registers.  The lanes, rows,
// chunks, reduction and every operation are the packed kernel's (16 lanes
// per row, 8 rows per lane group), so the results carry its bits.
constexpr int kStagedW = 4;  // warps per CTA: 64 rows of dk = 128

template <int DK, typename StT>
__host__ __device__ constexpr unsigned staged16_tile_bytes() {
  return (unsigned)(kStagedW * 2 * 8 * DK * sizeof(StT));
}

#ifndef GDN_STAGED_MIN_CTAS
#define GDN_STAGED_MIN_CTAS 8  // CTAs per SM the register budget is cut for (64 registers, no spills)
#endif

template <int DK, typename InT, typename OutT, typename StT>
__global__ void __launch_bounds__(kStagedW * 32, GDN_STAGED_MIN_CTAS)
    decode_staged16_kernel(const StepParams p) {
  constexpr int W = kStagedW, LPR = 16, M = 8, CW = 8;
  using L = Lanes<DK, LPR, CW>;
  static_assert(sizeof(StT) == 2 && DK == 128, "16-bit pools, dk = 128");
  constexpr int ROWS_W = L::GROUPS * M;
  constexpr int ROWS_CTA = W * ROWS_W;
  constexpr unsigned TILE_BYTES = staged16_tile_bytes<DK, StT>();
  static_assert(TILE_BYTES == ROWS_CTA * DK * sizeof(StT), "tile size");
  extern __shared__ __align__(128) unsigned char st16_smem[];
  const StT* Ss = reinterpret_cast<const StT*>(st16_smem);                 // [ROWS_CTA][DK]
  float* qk_s = reinterpret_cast<float*>(st16_smem + TILE_BYTES);          // k, q [DK] each, k.q
  __shared__ uint64_t bar;
  __shared__ int landed;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int pos = lane % LPR;
  const int bh = fdiv((int)blockIdx.x, p.div_tiles);
  const int tile = (int)blockIdx.x - bh * (int)p.div_tiles.d;
  const int b = fdiv(bh, p.div_h), h = bh - b * p.H;
  const int jl = warp * ROWS_W + (lane / LPR) * M;  // this group's first row in the tile
  const int j0 = tile * ROWS_CTA + jl;               // ... and in the head
  const int kh = fdiv(h, p.div_group);
  OutT* out = reinterpret_cast<OutT*>(p.out);

  // the token's inputs first (none depends on the slot): k and q (warp 0),
  // this group's v values and the gates; then the slot of the CTA
  // prefetch_ahead on, for the L2 prefetch of its tile
  float kv[DK / 32], qv[DK / 32];
  if (warp == 0) {
    const size_t base = ((size_t)b * p.Hk + kh) * DK;
    load_vec<InT, DK / 32>(reinterpret_cast<const InT*>(p.k) + base + lane * (DK / 32), kv);
    load_vec<InT, DK / 32>(reinterpret_cast<const InT*>(p.q) + base + lane * (DK / 32), qv);
  }
  float vv[M];
  load_vec<InT, M>(reinterpret_cast<const InT*>(p.v) + ((size_t)b * p.H + h) * p.dv + j0, vv);
  const float g_in = __ldg(p.g + (size_t)b * p.H + h);
  const float beta_in = __ldg(p.beta + (size_t)b * p.H + h);
  FutureTile fut{-1, 0, 0};
  if (threadIdx.x == (W - 1) * 32) fut = future_tile_begin(p);

  const int s = __ldg(p.slot_idx + b);
  if (s < 0 || (p.n_slots > 0 && s >= p.n_slots)) {
    if (s != -1 && p.dev_status != nullptr && lane == 0)
      atomicOr(p.dev_status, GDN_STATUS_SLOT_RANGE);
    if (pos < M) store_scalar(out + ((size_t)b * p.H + h) * p.dv + j0 + pos, 0.0f);
    return;
  }
  // where the state goes (one token): slot s, unless a commit of 0 tokens
  // keeps it, or a snapshot slot takes it
  int dst_slot = s;
  if (p.n_accept != nullptr) {
    const int n = __ldg(p.n_accept + b);
    if (n < 0 || n > 1) {
      if (p.dev_status != nullptr && lane == 0) atomicOr(p.dev_status, GDN_STATUS_ACCEPT_RANGE);
      dst_slot = -1;
    } else if (n == 0) {
      dst_slot = -1;
    }
  } else if (p.token_slots != nullptr) {
    dst_slot = __ldg(p.token_slots + b);
    if (dst_slot < -1 || (p.n_slots > 0 && dst_slot >= p.n_slots)) {
      if (p.dev_status != nullptr && lane == 0) atomicOr(p.dev_status, GDN_STATUS_SLOT_RANGE);
      dst_slot = -1;
    }
  }

  const size_t slot_stride = (size_t)p.H * p.dv * DK;
  const StT* src = reinterpret_cast<const StT*>(p.state) + (size_t)s * slot_stride +
                   ((size_t)h * p.dv + (size_t)tile * ROWS_CTA) * DK;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&bar, TILE_BYTES + kWaitTestExtraTx);
    bulk_copy_g2s(st16_smem, src, TILE_BYTES, &bar);
  }
  if (warp == 0)
    normalise_loaded<DK>(kv, qv, lane, p.l2_eps, p.l2norm, qk_s, qk_s + DK, qk_s + 2 * DK);
  TokenScalars ts;
  ts.scale = p.scale;
  ts.alpha = expf(g_in);
  ts.beta = beta_in;
  if (threadIdx.x == 0) landed = mbar_wait_bounded(&bar, 0, kWaitLimitNs) ? 1 : 0;
  __syncthreads();  // q, k normalised; the tile landed (or not)
  if (!landed) {
    // report, give the copy one more bounded wait so the shared memory is
    // not released under it, and leave the state as it was
    if (threadIdx.x == 0) {
      if (p.dev_status != nullptr) atomicOr(p.dev_status, GDN_STATUS_TIMEOUT);
      mbar_wait_bounded(&bar, 0, kWaitLimitNs);
    }
    return;
  }
  mbar_try_wait(&bar, 0);  // completed: every thread acquires the copied bytes
  ts.kq = qk_s[2 * DK];
  if (threadIdx.x == (W - 1) * 32) future_tile_prefetch<StT>(p, fut, ROWS_CTA, DK);

  // pass 1: S_m . k and S_m . q, in the packed kernel's order
  float red[2 * M];
#pragma unroll
  for (int m = 0; m < 2 * M; ++m) red[m] = 0.0f;
  const StT* row0 = Ss + (size_t)jl * DK;
#pragma unroll
  for (int c = 0; c < L::CH; ++c) {
    const float4 k0 = *reinterpret_cast<const float4*>(qk_s + L::offset(pos, c));
    const float4 k1 = *reinterpret_cast<const float4*>(qk_s + L::offset(pos, c) + 4);
    const float4 q0 = *reinterpret_cast<const float4*>(qk_s + DK + L::offset(pos, c));
    const float4 q1 = *reinterpret_cast<const float4*>(qk_s + DK + L::offset(pos, c) + 4);
    const float kc[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
    const float qc[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const uint4 t = *reinterpret_cast<const uint4*>(row0 + m * DK + L::offset(pos, c));
      const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float s0, s1;
        unpack2(StT(), w[i], s0, s1);
        red[m] = __fmaf_rn(s0, kc[2 * i], red[m]);
        red[M + m] = __fmaf_rn(s0, qc[2 * i], red[M + m]);
        red[m] = __fmaf_rn(s1, kc[2 * i + 1], red[m]);
        red[M + m] = __fmaf_rn(s1, qc[2 * i + 1], red[M + m]);
      }
    }
  }
  group_allreduce<LPR, 2 * M>(red);
  float d[M], o[M];
#pragma unroll
  for (int m = 0; m < M; ++m) {
    d[m] = __fmul_rn(ts.beta, __fsub_rn(vv[m], __fmul_rn(ts.alpha, red[m])));
    o[m] = __fmul_rn(ts.scale, __fmaf_rn(ts.kq, d[m], __fmul_rn(ts.alpha, red[M + m])));
  }
  const float mine = select_row<M>(o, pos);
  if (pos < M) store_scalar(out + ((size_t)b * p.H + h) * p.dv + j0 + pos, mine);

  // pass 2: the update in paired fp32 arithmetic, packed and stored
  if (dst_slot < 0) return;
  StT* dst = reinterpret_cast<StT*>(p.state) + (size_t)dst_slot * slot_stride +
             ((size_t)h * p.dv + j0) * DK;
  const uint64_t a2 = f32x2(ts.alpha, ts.alpha);
#pragma unroll
  for (int c = 0; c < L::CH; ++c) {
    const float4 k0 = *reinterpret_cast<const float4*>(qk_s + L::offset(pos, c));
    const float4 k1 = *reinterpret_cast<const float4*>(qk_s + L::offset(pos, c) + 4);
    const uint64_t kc2[4] = {f32x2(k0.x, k0.y), f32x2(k0.z, k0.w), f32x2(k1.x, k1.y),
                             f32x2(k1.z, k1.w)};
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const uint4 t = *reinterpret_cast<const uint4*>(row0 + m * DK + L::offset(pos, c));
      const uint32_t w[4] = {t.x, t.y, t.z, t.w};
      const uint64_t d2 = f32x2(d[m], d[m]);
      uint32_t r[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float s0, s1;
        unpack2(StT(), w[i], s0, s1);
        const uint64_t y = fma_f32x2(kc2[i], d2, mul_f32x2(a2, f32x2(s0, s1)));
        float y0, y1;
        split_f32x2(y, y0, y1);
        r[i] = pack2(StT(), y0, y1);
      }
      __stcs(reinterpret_cast<uint4*>(dst + (size_t)m * DK + L::offset(pos, c)),
             make_uint4(r[0], r[1], r[2], r[3]));
    }
  }
}

// ---------------------------------------------------------------------------
// the fused step: conv k=4 + SiLU, gates, recurrence, gated RMSNorm (T = 1)

struct FusedParams {
  const __nv_bfloat16* mixed_x;  // [B][C]
  __nv_bfloat16* conv_state;     // [n_slots][C][3]
  const void* conv_w;            // [C][4]
  const __nv_bfloat16* a;        // [B][H]
  const __nv_bfloat16* b;        // [B][H]
  const float* A_log;            // [H]
  const float* dt_bias;          // [H]
  const __nv_bfloat16* z;        // [B][H*dv]
  const float* norm_w;           // [dv]
  float* state;                  // [n_slots][H][dv][dk]
  const int32_t* slot_idx;       // [B]
  void* out;                     // [B][H][dv]
  int B, Hk, H, dv, n_slots, group, C;
  float norm_eps, scale, l2_eps;
  int* dev_status;
  FastDiv div_h, div_group;  // by H, by group (set at launch)
};

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + __expf(-x)); }

__device__ __forceinline__ float softplus_f(float x) {
  // log(1 + e^x) = max(x, 0) + log1p(e^-|x|)
  return fmaxf(x, 0.0f) + log1pf(__expf(-fabsf(x)));
}

__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
__device__ __forceinline__ unsigned cluster_ctarank() {
  unsigned r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}

// Grid: one CTA per (b, v-head h), blockIdx.x = b*H + h, launched in clusters
// of `group` = H/Hk CTAs: the v-heads that share one q/k head.  Every CTA of
// a cluster reads the old conv state of the shared q/k channels; the cluster
// barrier orders those reads before cluster rank 0 writes the shifted state.
// (The barrier is hardware: all CTAs of a cluster are co-resident and every
// thread arrives exactly once, so it always completes.)
template <int DK, int DV, int LPR, int M_MAX, int W, typename WT, typename OutT>
__global__ void __launch_bounds__(W * 32) fused_kernel(const FusedParams p) {
  using L = Lanes<DK, LPR, 4>;
  constexpr int EL = L::EL;
  constexpr int NT = W * 32;
  constexpr int ROWS_PER_WARP = DV / W;
  // rows per lane group: M_MAX, or fewer when a warp has fewer rows
  constexpr int M = ROWS_PER_WARP / L::GROUPS < M_MAX ? ROWS_PER_WARP / L::GROUPS : M_MAX;
  static_assert(M >= 1, "too few rows per warp for the lane groups");
  constexpr int ROWS_IT = L::GROUPS * M;  // rows a warp applies the token to at once
  constexpr int NG = ROWS_PER_WARP / ROWS_IT;
  static_assert(NG * ROWS_IT == ROWS_PER_WARP, "rows per warp must be a multiple of 32/LPR*M");
  constexpr int NCH = 2 * DK + DV;  // channels this CTA convolves
  constexpr int CPT = (NCH + NT - 1) / NT;

  __shared__ float qs[DK], ks[DK], vs[DV], os[DV], wsum[W];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int pos = lane % LPR;
  const int b = fdiv((int)blockIdx.x, p.div_h), h = (int)blockIdx.x - b * p.H;
  const int kh = fdiv(h, p.div_group);
  const bool writer = cluster_ctarank() == 0;
  OutT* out = reinterpret_cast<OutT*>(p.out);

  const int s = __ldg(p.slot_idx + b);
  if (s < 0 || s >= p.n_slots) {
    // the same decision is taken by every CTA of the cluster (same b), so
    // none of them enters the cluster barrier
    if (s != -1 && p.dev_status != nullptr && threadIdx.x == 0)
      atomicOr(p.dev_status, GDN_STATUS_SLOT_RANGE);
    for (int j = threadIdx.x; j < DV; j += NT)
      store_scalar(out + ((size_t)b * p.H + h) * DV + j, 0.0f);
    return;
  }

  // 1. start streaming the first row group of the state
  const int jw = warp * ROWS_PER_WARP + (lane / LPR) * M;  // this group's rows in iteration 0
  float* sp = p.state + (((size_t)s * p.H + h) * DV + jw) * DK;
  float S[M][EL], Sn[M][EL];
#pragma unroll
  for (int m = 0; m < M; ++m) load_row<float, DK, LPR>(sp + (size_t)m * DK, pos, S[m]);
  // the warp's later row groups (contiguous: rows warp*ROWS_PER_WARP + ROWS_IT
  // onwards) into L2, so that its row loop finds them there instead of
  // waiting on DRAM one row group at a time
  if (NG > 1 && lane == 0)
    prefetch_l2(p.state + (((size_t)s * p.H + h) * DV + warp * ROWS_PER_WARP + ROWS_IT) * DK,
                (unsigned)((ROWS_PER_WARP - ROWS_IT) * DK * sizeof(float)));

  // 2. conv k=4 + SiLU over this CTA's q, k and v channels
  const size_t cs_base = (size_t)s * p.C;
  float keep_x[CPT], keep_c1[CPT], keep_c2[CPT];
#pragma unroll
  for (int u = 0; u < CPT; ++u) {
    const int idx = threadIdx.x + u * NT;
    if (idx < NCH) {
      int c;
      if (idx < DK) c = kh * DK + idx;
      else if (idx < 2 * DK) c = p.Hk * DK + kh * DK + (idx - DK);
      else c = 2 * p.Hk * DK + h * DV + (idx - 2 * DK);
      const __nv_bfloat16* csp = p.conv_state + (cs_base + c) * 3;
      const float c0 = __bfloat162float(csp[0]);
      const float c1 = __bfloat162float(csp[1]);
      const float c2 = __bfloat162float(csp[2]);
      const float x = __bfloat162float(p.mixed_x[(size_t)b * p.C + c]);
      float w[4];
      load_vec<WT, 4>(reinterpret_cast<const WT*>(p.conv_w) + (size_t)c * 4, w);
      float y = __fmul_rn(w[0], c0);
      y = __fmaf_rn(w[1], c1, y);
      y = __fmaf_rn(w[2], c2, y);
      y = __fmaf_rn(w[3], x, y);
      y = silu_f(y);
      if (idx < DK) qs[idx] = y;
      else if (idx < 2 * DK) ks[idx - DK] = y;
      else vs[idx - 2 * DK] = y;
      keep_x[u] = x;
      keep_c1[u] = c1;
      keep_c2[u] = c2;
    }
  }
  // the v channels belong to this CTA alone: shift their conv state now
#pragma unroll
  for (int u = 0; u < CPT; ++u) {
    const int idx = threadIdx.x + u * NT;
    if (idx >= 2 * DK && idx < NCH) {
      const int c = 2 * p.Hk * DK + h * DV + (idx - 2 * DK);
      __nv_bfloat16* csp = p.conv_state + (cs_base + c) * 3;
      csp[0] = __float2bfloat16_rn(keep_c1[u]);
      csp[1] = __float2bfloat16_rn(keep_c2[u]);
      csp[2] = __float2bfloat16_rn(keep_x[u]);
    }
  }
  // this CTA has read the shared q/k conv state
  cluster_arrive_release();
  __syncthreads();

  // 3. gates, and this lane's elements of the normalised q and k (every warp
  //    sums |k|^2, |q|^2 and k.q over the shared-memory copies itself)
  TokenScalars ts;
  {
    const float A_log = __ldg(p.A_log + h);
    const float dtb = __ldg(p.dt_bias + h);
    const float av = __bfloat162float(p.a[(size_t)b * p.H + h]);
    const float bv = __bfloat162float(p.b[(size_t)b * p.H + h]);
    const float g = -__expf(A_log) * softplus_f(av + dtb);
    ts.alpha = __expf(g);
    ts.beta = 1.0f / (1.0f + __expf(-bv));
    ts.scale = p.scale;
  }
  float kn[EL], qn[EL];
  {
    constexpr int E = DK / 32;
    float red[3] = {0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float kx = ks[lane * E + e], qx = qs[lane * E + e];
      red[0] = __fmaf_rn(kx, kx, red[0]);
      red[1] = __fmaf_rn(qx, qx, red[1]);
      red[2] = __fmaf_rn(kx, qx, red[2]);
    }
    group_allreduce<32, 3>(red);
    const float rk = rsqrtf(__fadd_rn(red[0], p.l2_eps));
    const float rq = rsqrtf(__fadd_rn(red[1], p.l2_eps));
    ts.kq = __fmul_rn(__fmul_rn(red[2], rk), rq);
#pragma unroll
    for (int c = 0; c < L::CH; ++c)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        kn[4 * c + i] = __fmul_rn(ks[L::offset(pos, c) + i], rk);
        qn[4 * c + i] = __fmul_rn(qs[L::offset(pos, c) + i], rq);
      }
  }

  // 4. the recurrence over this warp's rows, ROWS_IT rows at a time, with
  //    the next rows' loads in flight
  float osq = 0.0f;
#pragma unroll
  for (int it = 0; it < NG; ++it) {
    if (it + 1 < NG) {
#pragma unroll
      for (int m = 0; m < M; ++m)
        load_row<float, DK, LPR>(sp + (size_t)((it + 1) * ROWS_IT + m) * DK, pos, Sn[m]);
    }
    const int jg = jw + it * ROWS_IT;
    float vv[M];
#pragma unroll
    for (int m = 0; m < M; ++m) vv[m] = vs[jg + m];
    float o[M];
    token_rows<LPR, EL, M, false>(S, kn, qn, vv, ts, o);
#pragma unroll
    for (int m = 0; m < M; ++m) {
      store_row<float, DK, LPR>(sp + (size_t)(it * ROWS_IT + m) * DK, pos, S[m]);
      osq = __fmaf_rn(o[m], o[m], osq);
    }
    const float mine = select_row<M>(o, pos);
    if (pos < M) os[jg + pos] = mine;
    if (it + 1 < NG) {
#pragma unroll
      for (int m = 0; m < M; ++m)
#pragma unroll
        for (int e = 0; e < EL; ++e) S[m][e] = Sn[m][e];
    }
  }
  // every lane of a group holds its group's sum: add the groups of the warp
#pragma unroll
  for (int off = 16; off >= LPR; off >>= 1) osq = __fadd_rn(osq, __shfl_xor_sync(kFull, osq, off));
  if (lane == 0) wsum[warp] = osq;
  __syncthreads();

  // 5. gated RMSNorm over the head's dv outputs
  float ss = 0.0f;
#pragma unroll
  for (int w = 0; w < W; ++w) ss = __fadd_rn(ss, wsum[w]);
  const float rinv = rsqrtf(__fadd_rn(__fdiv_rn(ss, (float)DV), p.norm_eps));
  for (int j = threadIdx.x; j < DV; j += NT) {
    const float zv = __bfloat162float(p.z[((size_t)b * p.H + h) * DV + j]);
    const float y = os[j] * rinv * __ldg(p.norm_w + j) * silu_f(zv);
    store_scalar(out + ((size_t)b * p.H + h) * DV + j, y);
  }

  // 6. every sibling has read the old q/k conv state: rank 0 shifts it
  cluster_wait_acquire();
  if (writer) {
#pragma unroll
    for (int u = 0; u < CPT; ++u) {
      const int idx = threadIdx.x + u * NT;
      if (idx < 2 * DK) {
        const int c = (idx < DK) ? kh * DK + idx : p.Hk * DK + kh * DK + (idx - DK);
        __nv_bfloat16* csp = p.conv_state + (cs_base + c) * 3;
        csp[0] = __float2bfloat16_rn(keep_c1[u]);
        csp[1] = __float2bfloat16_rn(keep_c2[u]);
        csp[2] = __float2bfloat16_rn(keep_x[u]);
      }
    }
  }
}

}  // namespace gdn
