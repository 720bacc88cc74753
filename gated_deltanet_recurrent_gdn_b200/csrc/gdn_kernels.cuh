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
//     differently in different instantiations: a T-token call is bit-identical
//     to T one-token calls.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

constexpr unsigned kFull = 0xffffffffu;

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

// The same placement applied to a dk-vector (q or k) of type In.
template <typename In, int DK, int LPR, int CW>
__device__ __forceinline__ void load_vec_lanes(const In* vec, int pos, float (&x)[DK / LPR]) {
  using L = Lanes<DK, LPR, CW>;
#pragma unroll
  for (int c = 0; c < L::CH; ++c) {
    float t[CW];
    load_vec<In, CW>(vec + L::offset(pos, c), t);
#pragma unroll
    for (int i = 0; i < CW; ++i) x[CW * c + i] = t[i];
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
  float l2_eps;
  int l2norm;
};

// Apply one token to the group's M rows S[m][0..EL) (this lane's elements)
// and return their outputs o_m (identical in every lane of the group).
//   kv, qv : this lane's elements of the raw k and q vectors
//   vv     : v_j of the group's M rows
template <int LPR, int EL, int M>
__device__ __forceinline__ void token_rows(float (&S)[M][EL], const float (&kv)[EL],
                                           const float (&qv)[EL], const float (&vv)[M],
                                           const TokenScalars& ts, float (&o)[M]) {
  // partial sums: [0]=|k|^2 [1]=|q|^2 [2]=k.q  [3+m]=S_m.k  [3+M+m]=S_m.q
  float red[3 + 2 * M];
  red[0] = __fmul_rn(kv[0], kv[0]);
  red[1] = __fmul_rn(qv[0], qv[0]);
  red[2] = __fmul_rn(kv[0], qv[0]);
#pragma unroll
  for (int e = 1; e < EL; ++e) {
    red[0] = __fmaf_rn(kv[e], kv[e], red[0]);
    red[1] = __fmaf_rn(qv[e], qv[e], red[1]);
    red[2] = __fmaf_rn(kv[e], qv[e], red[2]);
  }
#pragma unroll
  for (int m = 0; m < M; ++m) {
    float pk = __fmul_rn(S[m][0], kv[0]);
    float pq = __fmul_rn(S[m][0], qv[0]);
#pragma unroll
    for (int e = 1; e < EL; ++e) {
      pk = __fmaf_rn(S[m][e], kv[e], pk);
      pq = __fmaf_rn(S[m][e], qv[e], pq);
    }
    red[3 + m] = pk;
    red[3 + M + m] = pq;
  }
  group_allreduce<LPR, 3 + 2 * M>(red);

  float rk = 1.0f, rq = 1.0f;
  if (ts.l2norm) {
    rk = rsqrtf(__fadd_rn(red[0], ts.l2_eps));
    rq = rsqrtf(__fadd_rn(red[1], ts.l2_eps));
  }
  const float kq = __fmul_rn(__fmul_rn(red[2], rk), rq);  // (k/|k|).(q/|q|)
  float kn[EL];
#pragma unroll
  for (int e = 0; e < EL; ++e) kn[e] = __fmul_rn(kv[e], rk);

#pragma unroll
  for (int m = 0; m < M; ++m) {
    const float sk = __fmul_rn(red[3 + m], rk);      // (S^T k_hat)_j
    const float sq = __fmul_rn(red[3 + M + m], rq);  // (S^T q_hat)_j
    // delta = beta * (v - alpha * S^T k_hat)
    const float d = __fmul_rn(ts.beta, __fsub_rn(vv[m], __fmul_rn(ts.alpha, sk)));
    // o = scale * (alpha * S^T q_hat + (k_hat . q_hat) * delta)
    o[m] = __fmul_rn(ts.scale, __fmaf_rn(kq, d, __fmul_rn(ts.alpha, sq)));
    // S <- alpha * S + k_hat delta^T
#pragma unroll
    for (int e = 0; e < EL; ++e) S[m][e] = __fmaf_rn(kn[e], d, __fmul_rn(ts.alpha, S[m][e]));
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
};

// Grid: one CTA per (b, h, tile of W * 32/LPR * M rows); block: W warps.
// Block index order is tile fastest, then h, then b, so consecutive CTAs
// stream consecutive state memory of a slot.
template <int DK, int LPR, int M, int W, typename InT, typename OutT, typename StT>
__global__ void __launch_bounds__(W * 32) decode_kernel(const StepParams p) {
  constexpr int CW = StateTraits<StT>::CW;
  using L = Lanes<DK, LPR, CW>;
  constexpr int EL = L::EL;
  constexpr int ROWS_W = L::GROUPS * M;
  constexpr int ROWS_CTA = W * ROWS_W;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int pos = lane % LPR;
  const int tiles = p.dv / ROWS_CTA;
  int bid = blockIdx.x;
  const int tile = bid % tiles;
  bid /= tiles;
  const int h = bid % p.H;
  const int b = bid / p.H;
  const int j0 = tile * ROWS_CTA + warp * ROWS_W + (lane / LPR) * M;  // this group's rows
  const int kh = h / p.group;
  OutT* out = reinterpret_cast<OutT*>(p.out);

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

  StT* sp = reinterpret_cast<StT*>(p.state) + (((size_t)s * p.H + h) * p.dv + j0) * DK;
  float S[M][EL];
#pragma unroll
  for (int m = 0; m < M; ++m) load_row<StT, DK, LPR>(sp + (size_t)m * DK, pos, S[m]);

  TokenScalars ts;
  ts.scale = p.scale;
  ts.l2_eps = p.l2_eps;
  ts.l2norm = p.l2norm;
  for (int t = 0; t < p.T; ++t) {
    const size_t bt = (size_t)b * p.T + t;
    float kv[EL], qv[EL], vv[M];
    load_vec_lanes<InT, DK, LPR, CW>(reinterpret_cast<const InT*>(p.k) + (bt * p.Hk + kh) * DK, pos, kv);
    load_vec_lanes<InT, DK, LPR, CW>(reinterpret_cast<const InT*>(p.q) + (bt * p.Hk + kh) * DK, pos, qv);
    load_vec<InT, M>(reinterpret_cast<const InT*>(p.v) + (bt * p.H + h) * p.dv + j0, vv);
    ts.alpha = expf(__ldg(p.g + bt * p.H + h));
    ts.beta = __ldg(p.beta + bt * p.H + h);
    float o[M];
    token_rows<LPR, EL, M>(S, kv, qv, vv, ts, o);
    const float mine = select_row<M>(o, pos);
    if (pos < M) store_scalar(out + (bt * p.H + h) * p.dv + j0 + pos, mine);
  }

#pragma unroll
  for (int m = 0; m < M; ++m) store_row<StT, DK, LPR>(sp + (size_t)m * DK, pos, S[m]);
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
template <int DK, int DV, int LPR, int M, int W, typename WT, typename OutT>
__global__ void __launch_bounds__(W * 32) fused_kernel(const FusedParams p) {
  using L = Lanes<DK, LPR, 4>;
  constexpr int EL = L::EL;
  constexpr int NT = W * 32;
  constexpr int ROWS_PER_WARP = DV / W;
  constexpr int ROWS_IT = L::GROUPS * M;  // rows a warp applies the token to at once
  constexpr int NG = ROWS_PER_WARP / ROWS_IT;
  static_assert(NG * ROWS_IT == ROWS_PER_WARP, "rows per warp must be a multiple of 32/LPR*M");
  constexpr int NCH = 2 * DK + DV;  // channels this CTA convolves
  constexpr int CPT = (NCH + NT - 1) / NT;

  __shared__ float qs[DK], ks[DK], vs[DV], os[DV], wsum[W];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int pos = lane % LPR;
  const int h = blockIdx.x % p.H;
  const int b = blockIdx.x / p.H;
  const int kh = h / p.group;
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

  // 3. gates and this lane's elements of q, k
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
    ts.l2_eps = p.l2_eps;
    ts.l2norm = 1;
  }
  float kv[EL], qv[EL];
#pragma unroll
  for (int c = 0; c < L::CH; ++c)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      kv[4 * c + i] = ks[L::offset(pos, c) + i];
      qv[4 * c + i] = qs[L::offset(pos, c) + i];
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
    token_rows<LPR, EL, M>(S, kv, qv, vv, ts, o);
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
