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
// k and q vectors and [l*EV, l*EV+EV) of v, u and o.  The window (two
// contiguous blocks, R*dk and R*dv floats) is brought into shared memory by
// two bulk copies (cp.async.bulk, no multicast) that complete on the warp's
// mbarrier, so every byte of it is in flight at once.  Pass 1 sums both dot
// products of every entry (one reduce-scatter butterfly), pass 2 forms the
// prediction and the read-out from the u rows.  The new entry is written to
// shared memory (for the call's next token) and to the pool; the decay
// weights and the count are written once at the end.  HBM traffic per call
// is R*(dk+dv)*4 bytes read and T*(dk+dv)*4 + R*4 written per head.
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
  int prefetch_ahead;   // > 0: each warp asks L2 for the window of unit + this
};

// Warps (one per (sequence, head)) per CTA: each warp stages its window in
// shared memory, R*(dk+dv)*4 bytes, kept at 64 KB per CTA.
template <int DK, int DV, int R>
__host__ __device__ constexpr int lowrank_warps() {
  return (R * (DK + DV) * 4 * 4 <= 65536) ? 4 : (R * (DK + DV) * 4 * 2 <= 65536) ? 2 : 1;
}

template <int DK, int DV, int R>
__host__ __device__ constexpr size_t lowrank_smem_bytes() {
  return (size_t)lowrank_warps<DK, DV, R>() * R * (DK + DV) * 4 + 16 * lowrank_warps<DK, DV, R>();
}

// Reduce N values (16 <= N <= 128, a power of two) over the warp and scatter
// the sums: at each level of an xor butterfly a lane keeps one half of its
// vector (the upper half when its bit of the level is set) and adds the
// partner's copy of that half, so the vector halves each level.  Afterwards
// lane L holds the sums of values [L*N/32, (L+1)*N/32) in x[0..N/32); for
// N = 16 the pair of lanes 2i, 2i+1 both hold the sum of value i.
template <int N>
__device__ __forceinline__ void warp_reduce_scatter(float (&x)[N], int lane) {
  static_assert(N == 16 || N == 32 || N == 64 || N == 128, "N must be 16..128");
#pragma unroll
  for (int lvl = 0; lvl < 5; ++lvl) {
    const int o = 16 >> lvl;
    const int n = N >> lvl;  // values still held
    if (n >= 2) {
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < n / 2; ++i) {
        const float send = upper ? x[i] : x[i + n / 2];
        const float keep = upper ? x[i + n / 2] : x[i];
        x[i] = keep + __shfl_xor_sync(kFull, send, o);
      }
    } else {
      x[0] += __shfl_xor_sync(kFull, x[0], o);
    }
  }
}

template <int DK, int DV, int R, typename InT, typename OutT>
__global__ void __launch_bounds__(lowrank_warps<DK, DV, R>() * 32)
    lowrank_kernel(const LowrankParams p) {
  constexpr int W = lowrank_warps<DK, DV, R>();
  constexpr int E = DK / 32, EV = DV / 32;
  constexpr unsigned KB = R * DK * 4, UB = R * DV * 4;  // bytes of the two window blocks
  extern __shared__ __align__(128) float lr_smem[];
  __shared__ float sums[W][2 * R];  // the reduced dot products, per warp
  __shared__ uint64_t bars[W];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float* Ks = lr_smem + (size_t)warp * R * (DK + DV);  // [R][DK] cached k rows
  float* Us = Ks + R * DK;                             // [R][DV] cached u rows
  float* my_sums = sums[warp];
  uint64_t* bar = &bars[warp];
  const int unit = blockIdx.x * W + warp;
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

  // the whole window (two contiguous blocks) into shared memory, one copy
  // each, completing on this warp's mbarrier
  if (lane == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, KB + UB + kWaitTestExtraTx);
    bulk_copy_g2s(Ks, K, KB, bar);
    bulk_copy_g2s(Us, U, UB, bar);
  } else if (lane == 1 && p.prefetch_ahead > 0) {
    // the window of the unit about one wave of resident warps later, into L2
    const long long fut = (long long)unit + p.prefetch_ahead;
    if (fut < (long long)p.B * p.H) {
      const int fb = (int)(fut / p.H), fh = (int)(fut % p.H);
      const int fs = __ldg(p.slot_idx + fb);
      if (fs >= 0 && fs < p.n_slots) {
        const size_t fsh = (size_t)fs * p.H + fh;
        prefetch_l2(p.win_k + fsh * R * DK, KB);
        prefetch_l2(p.win_u + fsh * R * DV, UB);
      }
    }
  }
  // entries not yet made hold arbitrary bits: they are only ever selected
  // away, never multiplied in
  int count = *count_p;
  float cw0 = lane < R ? Cw[lane] : 0.0f;
  float cw1 = (R > 32) ? Cw[lane + 32] : 0.0f;
  __syncwarp();
  if (!mbar_wait_bounded(bar, 0, kWaitLimitNs)) {
    // the copy did not land: report, wait (bounded) for it once more so the
    // shared memory is not released under it, and leave the state as it was
    if (p.dev_status != nullptr && lane == 0) atomicOr(p.dev_status, GDN_STATUS_TIMEOUT);
    mbar_wait_bounded(bar, 0, kWaitLimitNs);
    return;
  }

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
    const int filled = count < R ? count : R;
    const int pos = count % R;  // ring position of the new update (the oldest when full)

    // decay weights: lane j holds c_j (and c_{j+32} for R = 64); entries
    // not yet made weigh 0 (their memory is not read as numbers)
    cw0 = (lane < filled) ? cw0 * alpha : 0.0f;
    cw1 = (R > 32 && lane + 32 < filled) ? cw1 * alpha : 0.0f;

    // pass 1: d_j = k_j . k and e_j = k_j . q, interleaved as red[2j], red[2j+1]
    float red[2 * R];
#pragma unroll
    for (int j = 0; j < R; ++j) {
      float kr[E];
      load_vec<float, E>(Ks + j * DK + lane * E, kr);
      float a = 0.0f, c = 0.0f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        a = fmaf(kr[e], kv[e], a);
        c = fmaf(kr[e], qv[e], c);
      }
      red[2 * j] = (j < filled) ? a : 0.0f;
      red[2 * j + 1] = (j < filled) ? c : 0.0f;
    }
    warp_reduce_scatter<2 * R>(red, lane);
    if constexpr (2 * R >= 32) {
#pragma unroll
      for (int i = 0; i < 2 * R / 32; ++i) my_sums[lane * (2 * R / 32) + i] = red[i];
    } else {
      my_sums[lane >> 1] = red[0];
    }
    __syncwarp();

    // pass 2: prediction and read-out sums over the u rows
    float pv[EV], ov[EV];
#pragma unroll
    for (int e = 0; e < EV; ++e) pv[e] = ov[e] = 0.0f;
#pragma unroll
    for (int j = 0; j < R; ++j) {
      const float cj = __shfl_sync(kFull, j < 32 ? cw0 : cw1, j & 31);
      float ur[EV];
      load_vec<float, EV>(Us + j * DV + lane * EV, ur);
      const float wp = cj * my_sums[2 * j];
      // the entry at `pos` is replaced when the window is full: it is not
      // part of the window the read-out sees
      const float wo = (filled == R && j == pos) ? 0.0f : cj * my_sums[2 * j + 1];
      if (j < filled) {
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
    // every lane has read the window and the sums: store the new entry in
    // shared memory (for the next token) and in the pool
    __syncwarp();
#pragma unroll
    for (int e = 0; e < E; ++e) {
      Ks[pos * DK + lane * E + e] = kv[e];
      K[(size_t)pos * DK + lane * E + e] = kv[e];
    }
#pragma unroll
    for (int e = 0; e < EV; ++e) {
      Us[pos * DV + lane * EV + e] = dlt[e];
      U[(size_t)pos * DV + lane * EV + e] = dlt[e];
    }
    if (lane == (pos & 31)) {
      if (pos < 32) cw0 = 1.0f;
      else cw1 = 1.0f;
    }
    ++count;
    __syncwarp();
  }
  // the decay weights and the count, once
  const int filled = count < R ? count : R;
  if (lane < filled) Cw[lane] = cw0;
  if (R > 32 && lane + 32 < filled) Cw[lane + 32] = cw1;
  if (lane == 0) *count_p = count;
}

}  // namespace gdn
