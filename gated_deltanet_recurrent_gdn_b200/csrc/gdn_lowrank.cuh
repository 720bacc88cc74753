// Low-rank sliding-window decode of the gated delta rule (sm_100a).
//
// The state of a head is a window of its R most recent rank-1 updates
// (k_j, u_j), each with the decay c_j accumulated since it was made; the
// state it stands for is S = sum_j c_j k_j u_j^T ("GDN tuning limits on
// Kunlun XPU", section 三.3: a sliding-window cache of the last r rank-1
// updates).  Per token:
//   c_j <- alpha c_j;  p = sum_j c_j (k_j . k) u_j;  delta = beta (v - p);
//   push (k, delta) with c = 1, replacing the oldest entry of a full window;
//   o = scale sum_{j in new window} c_j (k_j . q) u_j.
// Update number n (0-based) lives in ring position n % R.
//
// One warp per (sequence, head): lane l holds elements [l*E, l*E+E) of the
// k and q vectors and [l*EV, l*EV+EV) of v, u and o.  Pass 1 reads the
// window's k rows and sums both dot products of every entry in one batched
// butterfly; pass 2 reads the u rows once for the prediction and the
// read-out.  Only the new entry, the decay weights and the count are
// written, so HBM traffic per token is about R*(dk+dv)*4 bytes read and
// (dk+dv+R)*4 bytes written.
#pragma once

#include "gdn_kernels.cuh"

namespace gdn {

struct LowrankParams {
  const void* q;        // [B][T][Hk][dk]
  const void* k;        // [B][T][Hk][dk]
  const void* v;        // [B][T][H][dv]
  const float* g;       // [B][T][H]
  const float* beta;    // [B][T][H]
  float* win_k;         // [n_slots][H][R][dk]
  float* win_u;         // [n_slots][H][R][dv]
  float* win_c;         // [n_slots][H][R]
  int32_t* win_count;   // [n_slots][H]
  const int32_t* slot_idx;
  void* out;            // [B][T][H][dv]
  int B, T, Hk, H, n_slots, group;
  float scale, l2_eps;
  int l2norm;
  int* dev_status;
};

constexpr int kLowrankWarps = 4;

template <int DK, int DV, int R, typename InT, typename OutT>
__global__ void __launch_bounds__(kLowrankWarps * 32) lowrank_kernel(const LowrankParams p) {
  constexpr int E = DK / 32, EV = DV / 32;
  constexpr int G = R < 8 ? R : 8;  // window entries per pass-1 group
  static_assert(R % G == 0, "window length must be a multiple of the group");
  const int lane = threadIdx.x & 31;
  const int unit = blockIdx.x * kLowrankWarps + (threadIdx.x >> 5);
  if (unit >= p.B * p.H) return;  // whole warps only: no warp-collective below is split
  const int b = unit / p.H, h = unit % p.H, kh = h / p.group;
  OutT* out = reinterpret_cast<OutT*>(p.out);

  const int s = __ldg(p.slot_idx + b);
  if (s < 0 || s >= p.n_slots) {
    if (s != -1 && p.dev_status != nullptr && lane == 0)
      atomicOr(p.dev_status, GDN_STATUS_SLOT_RANGE);
    for (int t = 0; t < p.T; ++t)
#pragma unroll
      for (int e = 0; e < EV; ++e)
        store_scalar(out + (((size_t)b * p.T + t) * p.H + h) * DV + lane * EV + e, 0.0f);
    return;
  }
  const size_t sh = (size_t)s * p.H + h;
  float* K = p.win_k + sh * R * DK;
  float* U = p.win_u + sh * R * DV;
  float* Cw = p.win_c + sh * R;
  int32_t* count_p = p.win_count + sh;

  for (int t = 0; t < p.T; ++t) {
    const size_t bt = (size_t)b * p.T + t;
    // normalised q, k (this lane's elements), v, gates
    float kv[E], qv[E], vv[EV];
    load_vec<InT, E>(reinterpret_cast<const InT*>(p.k) + (bt * p.Hk + kh) * DK + lane * E, kv);
    load_vec<InT, E>(reinterpret_cast<const InT*>(p.q) + (bt * p.Hk + kh) * DK + lane * E, qv);
    load_vec<InT, EV>(reinterpret_cast<const InT*>(p.v) + (bt * p.H + h) * DV + lane * EV, vv);
    float nrm[3] = {0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int e = 0; e < E; ++e) {
      nrm[0] = fmaf(kv[e], kv[e], nrm[0]);
      nrm[1] = fmaf(qv[e], qv[e], nrm[1]);
      nrm[2] = fmaf(kv[e], qv[e], nrm[2]);
    }
    group_allreduce<32, 3>(nrm);
    const float rk = p.l2norm ? rsqrtf(nrm[0] + p.l2_eps) : 1.0f;
    const float rq = p.l2norm ? rsqrtf(nrm[1] + p.l2_eps) : 1.0f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      kv[e] *= rk;
      qv[e] *= rq;
    }
    const float kq = nrm[2] * rk * rq;
    const float alpha = expf(__ldg(p.g + bt * p.H + h));
    const float beta = __ldg(p.beta + bt * p.H + h);
    const int count = *count_p;
    const int filled = count < R ? count : R;
    const int pos = count % R;  // ring position of the new update (the oldest when full)

    // decay weights: lane j holds c_j (R <= 64: two per lane at most)
    float cw0 = (lane < filled) ? Cw[lane] * alpha : 0.0f;
    float cw1 = (R > 32 && lane + 32 < filled) ? Cw[lane + 32] * alpha : 0.0f;

    // pass 1: d_j = k_j . k and e_j = k_j . q for every entry
    float dkj[R], dqj[R];
#pragma unroll
    for (int g0 = 0; g0 < R; g0 += G) {
      float kr[G][E];
#pragma unroll
      for (int j = 0; j < G; ++j) {
        if (g0 + j < filled) {
          load_vec<float, E>(K + (size_t)(g0 + j) * DK + lane * E, kr[j]);
        } else {
#pragma unroll
          for (int e = 0; e < E; ++e) kr[j][e] = 0.0f;
        }
      }
#pragma unroll
      for (int j = 0; j < G; ++j) {
        float a = 0.0f, c = 0.0f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          a = fmaf(kr[j][e], kv[e], a);
          c = fmaf(kr[j][e], qv[e], c);
        }
        dkj[g0 + j] = a;
        dqj[g0 + j] = c;
      }
    }
    group_allreduce<32, R>(dkj);
    group_allreduce<32, R>(dqj);

    // pass 2: prediction and read-out sums over the u rows
    float pv[EV], ov[EV];
#pragma unroll
    for (int e = 0; e < EV; ++e) pv[e] = ov[e] = 0.0f;
#pragma unroll
    for (int j = 0; j < R; ++j) {
      if (j < filled) {
        const float cj = __shfl_sync(kFull, j < 32 ? cw0 : cw1, j & 31);
        float ur[EV];
        load_vec<float, EV>(U + (size_t)j * DV + lane * EV, ur);
        const float wp = cj * dkj[j];
        // the entry at `pos` is replaced when the window is full: it is not
        // part of the window the read-out sees
        const float wo = (filled == R && j == pos) ? 0.0f : cj * dqj[j];
#pragma unroll
        for (int e = 0; e < EV; ++e) {
          pv[e] = fmaf(wp, ur[e], pv[e]);
          ov[e] = fmaf(wo, ur[e], ov[e]);
        }
      }
    }
    float dlt[EV];
#pragma unroll
    for (int e = 0; e < EV; ++e) {
      dlt[e] = beta * (vv[e] - pv[e]);
      const float o = p.scale * fmaf(kq, dlt[e], ov[e]);
      store_scalar(out + (bt * p.H + h) * DV + lane * EV + e, o);
    }
    // every lane has read the window: write the new entry, weights, count
    __syncwarp();
#pragma unroll
    for (int e = 0; e < E; ++e) K[(size_t)pos * DK + lane * E + e] = kv[e];
#pragma unroll
    for (int e = 0; e < EV; ++e) U[(size_t)pos * DV + lane * EV + e] = dlt[e];
    if (lane < filled) Cw[lane] = cw0;
    if (R > 32 && lane + 32 < filled) Cw[lane + 32] = cw1;
    if (lane == (pos & 31)) Cw[pos] = 1.0f;
    if (lane == 0) *count_p = count + 1;
    __syncwarp();
    __threadfence_block();  // the next token of this warp reads what was just written
  }
}

}  // namespace gdn
