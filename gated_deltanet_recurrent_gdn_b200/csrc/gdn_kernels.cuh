// Device side of the gated delta rule decode library (sm_100a).
//
// The decode step is HBM-bound: per (sequence, head) the dk x dv fp32 state
// is read once and written once, and the arithmetic is two mat-vec products
// and a rank-1 update (about 7 flop per 8 bytes of state), so there is no
// dense contraction for the tensor cores.  The kernels below are built as a
// stream over state rows:
//
//   * A state row is one dv column of S: dk contiguous floats (512 B for
//     dk = 128).  A warp owns whole rows; lane l holds elements
//     [l*E, l*E + E) of each of its R rows (E = dk/32), so every row is one
//     fully coalesced 128-bit-per-lane load and store.
//   * Per token, both dot products S^T k and S^T q of every row, plus the
//     three scalars |k|^2, |q|^2 and k.q needed for the L2 norms, are summed
//     in ONE warp butterfly (all lanes end with every sum, bit-identical).
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
    static_assert(BYTES == 32, "unsupported vector size");
    uint4 t0 = reinterpret_cast<const uint4*>(p)[0];
    uint4 t1 = reinterpret_cast<const uint4*>(p)[1];
    w[0] = t0.x; w[1] = t0.y; w[2] = t0.z; w[3] = t0.w;
    w[4] = t1.x; w[5] = t1.y; w[6] = t1.z; w[7] = t1.w;
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

// State rows: E fp32 per lane.  Streaming (evict-first) hints keep the
// once-touched state from displacing the small per-token inputs in L2.
template <int E>
__device__ __forceinline__ void load_state(const float* p, float (&s)[E]) {
  if constexpr (E == 4) {
    float4 t = __ldcs(reinterpret_cast<const float4*>(p));
    s[0] = t.x; s[1] = t.y; s[2] = t.z; s[3] = t.w;
  } else {
    static_assert(E == 2, "dk must be 64 or 128");
    float2 t = __ldcs(reinterpret_cast<const float2*>(p));
    s[0] = t.x; s[1] = t.y;
  }
}

template <int E>
__device__ __forceinline__ void store_state(float* p, const float (&s)[E]) {
  if constexpr (E == 4) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(s[0], s[1], s[2], s[3]));
  } else {
    __stcs(reinterpret_cast<float2*>(p), make_float2(s[0], s[1]));
  }
}

// All-reduce N values over the warp with an xor butterfly.  Every lane ends
// with the same bits (each partner pair adds the same two operands).
template <int N>
__device__ __forceinline__ void warp_allreduce(float (&x)[N]) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
#pragma unroll
    for (int i = 0; i < N; ++i) x[i] = __fadd_rn(x[i], __shfl_xor_sync(kFull, x[i], off));
  }
}

// ---------------------------------------------------------------------------
// one token on R rows held by a warp

struct TokenScalars {
  float alpha;  // exp(g)
  float beta;
  float scale;
  float l2_eps;
  int l2norm;
};

// Apply one token to the warp's R rows S[r][0..E) (this lane's slice) and
// return the R outputs o_r (identical in every lane).
//   kv, qv : this lane's slice of the raw k and q vectors (dk elements total)
//   vv     : the R values v_j of the warp's rows
template <int E, int R>
__device__ __forceinline__ void token_rows(float (&S)[R][E], const float (&kv)[E],
                                           const float (&qv)[E], const float (&vv)[R],
                                           const TokenScalars& ts, float (&o)[R]) {
  // partial sums: [0]=|k|^2 [1]=|q|^2 [2]=k.q  [3+r]=S_r.k  [3+R+r]=S_r.q
  float red[3 + 2 * R];
  red[0] = __fmul_rn(kv[0], kv[0]);
  red[1] = __fmul_rn(qv[0], qv[0]);
  red[2] = __fmul_rn(kv[0], qv[0]);
#pragma unroll
  for (int e = 1; e < E; ++e) {
    red[0] = __fmaf_rn(kv[e], kv[e], red[0]);
    red[1] = __fmaf_rn(qv[e], qv[e], red[1]);
    red[2] = __fmaf_rn(kv[e], qv[e], red[2]);
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float pk = __fmul_rn(S[r][0], kv[0]);
    float pq = __fmul_rn(S[r][0], qv[0]);
#pragma unroll
    for (int e = 1; e < E; ++e) {
      pk = __fmaf_rn(S[r][e], kv[e], pk);
      pq = __fmaf_rn(S[r][e], qv[e], pq);
    }
    red[3 + r] = pk;
    red[3 + R + r] = pq;
  }
  warp_allreduce<3 + 2 * R>(red);

  float rk = 1.0f, rq = 1.0f;
  if (ts.l2norm) {
    rk = rsqrtf(__fadd_rn(red[0], ts.l2_eps));
    rq = rsqrtf(__fadd_rn(red[1], ts.l2_eps));
  }
  const float kq = __fmul_rn(__fmul_rn(red[2], rk), rq);  // (k/|k|).(q/|q|)
  float kn[E];
#pragma unroll
  for (int e = 0; e < E; ++e) kn[e] = __fmul_rn(kv[e], rk);

#pragma unroll
  for (int r = 0; r < R; ++r) {
    const float sk = __fmul_rn(red[3 + r], rk);      // (S^T k_hat)_j
    const float sq = __fmul_rn(red[3 + R + r], rq);  // (S^T q_hat)_j
    // delta = beta * (v - alpha * S^T k_hat)
    const float d = __fmul_rn(ts.beta, __fsub_rn(vv[r], __fmul_rn(ts.alpha, sk)));
    // o = scale * (alpha * S^T q_hat + (k_hat . q_hat) * delta)
    o[r] = __fmul_rn(ts.scale, __fmaf_rn(kq, d, __fmul_rn(ts.alpha, sq)));
    // S <- alpha * S + k_hat delta^T
#pragma unroll
    for (int e = 0; e < E; ++e) S[r][e] = __fmaf_rn(kn[e], d, __fmul_rn(ts.alpha, S[r][e]));
  }
}

// lane r (< R) picks o[r]; other lanes get o[0] (unused)
template <int R>
__device__ __forceinline__ float select_lane(const float (&o)[R], int lane) {
  float x = o[0];
#pragma unroll
  for (int r = 1; r < R; ++r) x = (lane == r) ? o[r] : x;
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
  float* state;
  const int32_t* slot_idx;
  void* out;
  int B, Hk, H, dv, T, n_slots, group;
  float scale, l2_eps;
  int l2norm;
  int* dev_status;
};

// Grid: one CTA per (b, h, tile of W*R rows); block: W warps.  Block index
// order is tile fastest, then h, then b, so consecutive CTAs stream
// consecutive state memory of a slot.
template <int DK, int R, int W, typename InT, typename OutT>
__global__ void __launch_bounds__(W * 32) decode_kernel(const StepParams p) {
  constexpr int E = DK / 32;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int tiles = p.dv / (W * R);
  int bid = blockIdx.x;
  const int tile = bid % tiles;
  bid /= tiles;
  const int h = bid % p.H;
  const int b = bid / p.H;
  const int j0 = (tile * W + warp) * R;
  const int kh = h / p.group;
  OutT* out = reinterpret_cast<OutT*>(p.out);

  const int s = __ldg(p.slot_idx + b);
  if (s < 0 || (p.n_slots > 0 && s >= p.n_slots)) {
    if (s != -1 && p.dev_status != nullptr && lane == 0)
      atomicOr(p.dev_status, GDN_STATUS_SLOT_RANGE);
    if (lane < R) {
      for (int t = 0; t < p.T; ++t)
        store_scalar(out + (((size_t)b * p.T + t) * p.H + h) * p.dv + j0 + lane, 0.0f);
    }
    return;
  }

  float* sp = p.state + (((size_t)s * p.H + h) * p.dv + j0) * DK + lane * E;
  float S[R][E];
#pragma unroll
  for (int r = 0; r < R; ++r) load_state<E>(sp + (size_t)r * DK, S[r]);

  TokenScalars ts;
  ts.scale = p.scale;
  ts.l2_eps = p.l2_eps;
  ts.l2norm = p.l2norm;
  for (int t = 0; t < p.T; ++t) {
    const size_t bt = (size_t)b * p.T + t;
    float kv[E], qv[E], vv[R];
    load_vec<InT, E>(reinterpret_cast<const InT*>(p.k) + (bt * p.Hk + kh) * DK + lane * E, kv);
    load_vec<InT, E>(reinterpret_cast<const InT*>(p.q) + (bt * p.Hk + kh) * DK + lane * E, qv);
    load_vec<InT, R>(reinterpret_cast<const InT*>(p.v) + (bt * p.H + h) * p.dv + j0, vv);
    ts.alpha = expf(__ldg(p.g + bt * p.H + h));
    ts.beta = __ldg(p.beta + bt * p.H + h);
    float o[R];
    token_rows<E, R>(S, kv, qv, vv, ts, o);
    const float mine = select_lane<R>(o, lane);
    if (lane < R) store_scalar(out + (bt * p.H + h) * p.dv + j0 + lane, mine);
  }

#pragma unroll
  for (int r = 0; r < R; ++r) store_state<E>(sp + (size_t)r * DK, S[r]);
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
template <int DK, int DV, int W, int R, typename WT, typename OutT>
__global__ void __launch_bounds__(W * 32) fused_kernel(const FusedParams p) {
  constexpr int E = DK / 32;
  constexpr int NT = W * 32;
  constexpr int ROWS_PER_WARP = DV / W;
  constexpr int NG = ROWS_PER_WARP / R;
  static_assert(ROWS_PER_WARP % R == 0, "rows per warp must be a multiple of R");
  constexpr int NCH = 2 * DK + DV;  // channels this CTA convolves
  constexpr int CPT = (NCH + NT - 1) / NT;

  __shared__ float qs[DK], ks[DK], vs[DV], os[DV], wsum[W];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
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
  float* sp = p.state + (((size_t)s * p.H + h) * DV + warp * ROWS_PER_WARP) * DK + lane * E;
  float S[R][E], Sn[R][E];
#pragma unroll
  for (int r = 0; r < R; ++r) load_state<E>(sp + (size_t)r * DK, S[r]);

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

  // 3. gates and per-warp copies of q, k
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
  float kv[E], qv[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    kv[e] = ks[lane * E + e];
    qv[e] = qs[lane * E + e];
  }

  // 4. the recurrence over this warp's rows, one group of R rows at a time,
  //    with the next group's loads in flight
  float osq = 0.0f;
#pragma unroll
  for (int grp = 0; grp < NG; ++grp) {
    if (grp + 1 < NG) {
#pragma unroll
      for (int r = 0; r < R; ++r)
        load_state<E>(sp + (size_t)((grp + 1) * R + r) * DK, Sn[r]);
    }
    const int jg = warp * ROWS_PER_WARP + grp * R;
    float vv[R];
#pragma unroll
    for (int r = 0; r < R; ++r) vv[r] = vs[jg + r];
    float o[R];
    token_rows<E, R>(S, kv, qv, vv, ts, o);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      store_state<E>(sp + (size_t)(grp * R + r) * DK, S[r]);
      osq = __fmaf_rn(o[r], o[r], osq);
    }
    const float mine = select_lane<R>(o, lane);
    if (lane < R) os[jg + lane] = mine;
    if (grp + 1 < NG) {
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int e = 0; e < E; ++e) S[r][e] = Sn[r][e];
    }
  }
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
