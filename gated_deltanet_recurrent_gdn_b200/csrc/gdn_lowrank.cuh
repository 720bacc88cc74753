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
// Each (sequence, head) is handled by S = max(1, R / 16) warps, each owning
// E = R / S consecutive ring positions of the window (at most 16), so that
// no warp carries more than 16 entries through its dependent chain.  Lane l
// holds elements [l*E32, l*E32+E32) of the k and q vectors and
// [l*EV, l*EV+EV) of v, u and o.  A warp brings its slice of the window (two
// contiguous blocks, E*dk and E*dv floats) into shared memory with two bulk
// copies (cp.async.bulk, no multicast) on its own mbarrier, so every byte is
// in flight at once.  Per token, pass 1 sums both dot products of each of
// its entries (one reduce-scatter butterfly), pass 2 its share of the
// prediction and the read-out from its u rows; with S > 1 the S partial
// vectors meet in shared memory (one named barrier per token) and every
// warp of the head adds them in the same order.  The warp that owns the
// ring position of the new entry writes it to shared memory (for the call's
// next token) and to the pool; decay weights and the count are written once
// at the end.  HBM traffic per call is R*(dk+dv)*4 bytes read and
// T*(dk+dv)*4 + R*4 written per head.
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
  int prefetch_ahead;   // one wave of resident units; each warp asks L2 for the
                        // window of unit + half of it
  FastDiv div_h, div_group;  // by H, by group (set at launch)
};

// Window entries per warp at most (a power of two, 8 or 16).
#ifndef GDN_LOWRANK_ENTRIES
#define GDN_LOWRANK_ENTRIES 16
#endif

// Warps per (sequence, head): at most GDN_LOWRANK_ENTRIES window entries per warp.
template <int R>
__host__ __device__ constexpr int lowrank_split() {
  return R > GDN_LOWRANK_ENTRIES ? R / GDN_LOWRANK_ENTRIES : 1;
}

// Shared memory a CTA stages windows in, at most (one unit's window always
// fits).  Smaller CTAs finish independently: with dk = dv = 128 every window
// of 8 or more entries is a CTA of its own, which measured 2% (32 entries),
// 7% (16) and 8% (8) faster than two to four windows per 64 KB CTA.
#ifndef GDN_LOWRANK_CTA_BYTES
#define GDN_LOWRANK_CTA_BYTES 8192
#endif

// Warps per CTA: (sequence, head) units of lowrank_split warps each, with
// their windows, R*(dk+dv)*4 bytes per unit, staged in at most
// GDN_LOWRANK_CTA_BYTES.
template <int DK, int DV, int R>
__host__ __device__ constexpr int lowrank_warps() {
  constexpr int unit_bytes = R * (DK + DV) * 4;
  constexpr int cta = GDN_LOWRANK_CTA_BYTES;
  constexpr int units = unit_bytes * 4 <= cta ? 4 : unit_bytes * 2 <= cta ? 2 : 1;
  return units * lowrank_split<R>() > 8 ? 8 : units * lowrank_split<R>();
}

// Dynamic shared memory: the windows, then the partial prediction and
// read-out vectors of the split units ([warp][token parity][2][DV]).
template <int DK, int DV, int R>
__host__ __device__ constexpr size_t lowrank_smem_bytes() {
  return (size_t)(lowrank_warps<DK, DV, R>() / lowrank_split<R>()) * R * (DK + DV) * 4 +
         (lowrank_split<R>() > 1 ? (size_t)lowrank_warps<DK, DV, R>() * 2 * 2 * DV * 4 : 0);
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

// The named barrier of the S warps of unit `ul` (ids 1..UPC; 0 is the
// CTA-wide barrier).  The id is a constant in every branch, so the kernel
// reserves only the barriers it names.
template <int S, int UPC>
__device__ __forceinline__ void unit_barrier(int ul) {
  static_assert(UPC <= 8, "at most 8 units per CTA");
#define GDN_UNIT_BAR(ID)                                                             \
  if (ul == ID - 1) {                                                                \
    asm volatile("bar.sync %0, %1;\n" ::"n"(ID), "n"(S * 32) : "memory");           \
    return;                                                                          \
  }
  GDN_UNIT_BAR(1)
  if constexpr (UPC > 1) { GDN_UNIT_BAR(2) }
  if constexpr (UPC > 2) { GDN_UNIT_BAR(3) GDN_UNIT_BAR(4) }
  if constexpr (UPC > 4) { GDN_UNIT_BAR(5) GDN_UNIT_BAR(6) GDN_UNIT_BAR(7) GDN_UNIT_BAR(8) }
#undef GDN_UNIT_BAR
}

template <int DK, int DV, int R, typename InT, typename OutT>
__global__ void __launch_bounds__(lowrank_warps<DK, DV, R>() * 32)
    lowrank_kernel(const LowrankParams p) {
  constexpr int W = lowrank_warps<DK, DV, R>();
  constexpr int S = lowrank_split<R>();   // warps per (sequence, head)
  constexpr int UPC = W / S;              // (sequence, head) units per CTA
  constexpr int E = R / S;                // window entries per warp
  constexpr int E32 = DK / 32, EV = DV / 32;
  constexpr unsigned KB = E * DK * 4, UB = E * DV * 4;  // bytes of a warp's two blocks
  static_assert(W % S == 0 && E <= 32 && (2 * E == 16 || 2 * E == 32), "window split");
  extern __shared__ __align__(128) float lr_smem[];
  __shared__ float sums[W][2 * E];  // the reduced dot products, per warp
  __shared__ uint64_t bars[W];
  __shared__ int landed_s[W];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ul = warp / S, wu = warp % S;  // unit within the CTA, warp within the unit
  // this warp's slice of its unit's window: [E][DK] cached k rows, [E][DV] u rows
  float* Ks = lr_smem + (size_t)ul * R * (DK + DV) + (size_t)wu * E * (DK + DV);
  float* Us = Ks + E * DK;
  // partial prediction and read-out vectors: [warp][token parity][2][DV]
  float* part = lr_smem + (size_t)UPC * R * (DK + DV);
  float* my_sums = sums[warp];
  uint64_t* bar = &bars[warp];
  const int unit = blockIdx.x * UPC + ul;
  if (unit >= p.B * p.H) return;  // whole units only: no barrier below is split
  const int b = fdiv(unit, p.div_h), h = unit - b * p.H, kh = fdiv(h, p.div_group);
  OutT* out = reinterpret_cast<OutT*>(p.out);

  // The first token's inputs are requested before the slot, which none of
  // them depends on; lanes 1 and 2 also request the slot of the unit about
  // one wave of resident units on, for the L2 prefetch below (so that the
  // warp does not wait for it there).
  float kv0[E32], qv0[E32], vv0[EV];
  {
    const size_t bt = (size_t)b * p.T;
    load_vec<InT, E32>(reinterpret_cast<const InT*>(p.k) + (bt * p.Hk + kh) * DK + lane * E32, kv0);
    load_vec<InT, E32>(reinterpret_cast<const InT*>(p.q) + (bt * p.Hk + kh) * DK + lane * E32, qv0);
    load_vec<InT, EV>(reinterpret_cast<const InT*>(p.v) + (bt * p.H + h) * DV + lane * EV, vv0);
  }
  const float g0 = __ldg(p.g + (size_t)b * p.T * p.H + h);
  const float beta0 = __ldg(p.beta + (size_t)b * p.T * p.H + h);
  // half of the launcher's one wave (measured at R = 8, 16, 32: 23.5 -> 22.7,
  // 38.4 -> 37.3, 69.1 -> 66.8 us per launch against a whole wave)
  const long long fut = (long long)unit + p.prefetch_ahead / 2;
  const bool fut_ok = p.prefetch_ahead > 1 && fut < (long long)p.B * p.H;
  const int fb = fut_ok ? fdiv((int)fut, p.div_h) : 0;
  const int fh = fut_ok ? (int)fut - fb * p.H : 0;
  int fs = -1;
  if (fut_ok && lane >= 1 && lane <= 2) fs = __ldg(p.slot_idx + fb);

  const int s = __ldg(p.slot_idx + b);
  if (s < 0 || s >= p.n_slots) {
    if (wu == 0) {
      if (s != -1 && p.dev_status != nullptr && lane == 0)
        atomicOr(p.dev_status, GDN_STATUS_SLOT_RANGE);
      for (int t = 0; t < p.T; ++t)
#pragma unroll
        for (int e = 0; e < EV; ++e)
          store_scalar(out + (((size_t)b * p.T + t) * p.H + h) * DV + lane * EV + e, 0.0f);
    }
    return;
  }
  const size_t sh = (size_t)s * p.H + h;
  float* K = p.win_k + sh * R * DK;
  float* U = p.win_u + sh * R * DV;
  float* Cw = p.win_c + sh * R;
  int32_t* count_p = p.win_count + sh;
  const int j0 = wu * E;  // this warp's first ring position

  // this warp's slice of the window (two contiguous blocks) into shared
  // memory, one copy each, completing on this warp's mbarrier
  if (lane == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, KB + UB + kWaitTestExtraTx);
    bulk_copy_g2s(Ks, K + (size_t)j0 * DK, KB, bar);
    bulk_copy_g2s(Us, U + (size_t)j0 * DV, UB, bar);
  } else if (lane <= 4 && fut_ok) {
    // for the unit about one wave of resident units later, into L2: lane 1
    // the same slice of its window, lane 2 this slice's decay weights and
    // the count, lane 3 of the unit's first warp its first token's q and k
    // rows, lane 4 of its last warp the v row, gate and beta (the loads
    // that open that unit's dependent chain)
    {
      const size_t bt = (size_t)fb * p.T;
      if (lane <= 2) {
        if (fs >= 0 && fs < p.n_slots) {
          const size_t fsh = (size_t)fs * p.H + fh;
          if (lane == 1) {
            prefetch_l2(p.win_k + fsh * R * DK + (size_t)j0 * DK, KB);
            prefetch_l2(p.win_u + fsh * R * DV + (size_t)j0 * DV, UB);
          } else {
            prefetch_l2_line(p.win_c + fsh * R + j0);
            prefetch_l2_line(p.win_count + fsh);
          }
        }
      } else if (lane == 3 && wu == 0) {
        const size_t row = (bt * p.Hk + fdiv(fh, p.div_group)) * DK;
        prefetch_l2(reinterpret_cast<const InT*>(p.q) + row, DK * sizeof(InT));
        prefetch_l2(reinterpret_cast<const InT*>(p.k) + row, DK * sizeof(InT));
      } else if (lane == 4 && wu == S - 1) {
        prefetch_l2(reinterpret_cast<const InT*>(p.v) + (bt * p.H + fh) * DV, DV * sizeof(InT));
        prefetch_l2_line(p.g + bt * p.H + fh);
        prefetch_l2_line(p.beta + bt * p.H + fh);
      }
    }
  }
  // entries not yet made hold arbitrary bits: they are only ever selected
  // away, never multiplied in.  Lane l < E holds c of ring position j0 + l.
  int count = *count_p;
  float cw = lane < E ? Cw[j0 + lane] : 0.0f;
  __syncwarp();
  bool landed = mbar_wait_bounded(bar, 0, kWaitLimitNs);
  if constexpr (S > 1) {
    // the warps of a unit decide together, so that none of them waits at
    // the unit's named barrier below for a warp that has returned: every
    // warp reaches this barrier exactly once, after its bounded wait
    if (lane == 0) landed_s[warp] = landed ? 1 : 0;
    unit_barrier<S, UPC>(ul);
    bool all = true;
#pragma unroll
    for (int w2 = 0; w2 < S; ++w2) all = all && landed_s[ul * S + w2] != 0;
    if (landed && !all) return;  // this warp's copy has landed; another's has not
  }
  if (!landed) {
    // the copy did not land: report, wait (bounded) for it once more so the
    // shared memory is not released under it, and leave the state as it was
    if (p.dev_status != nullptr && lane == 0) atomicOr(p.dev_status, GDN_STATUS_TIMEOUT);
    mbar_wait_bounded(bar, 0, kWaitLimitNs);
    return;
  }

  for (int t = 0; t < p.T; ++t) {
    const size_t bt = (size_t)b * p.T + t;
    // normalised q, k (this lane's elements), v, gates (every warp of the
    // unit); the first token's were loaded at the start
    float kv[E32], qv[E32], vv[EV];
    float g_t = g0, beta_t = beta0;
    if (t == 0) {
#pragma unroll
      for (int e = 0; e < E32; ++e) {
        kv[e] = kv0[e];
        qv[e] = qv0[e];
      }
#pragma unroll
      for (int e = 0; e < EV; ++e) vv[e] = vv0[e];
    } else {
      load_vec<InT, E32>(reinterpret_cast<const InT*>(p.k) + (bt * p.Hk + kh) * DK + lane * E32, kv);
      load_vec<InT, E32>(reinterpret_cast<const InT*>(p.q) + (bt * p.Hk + kh) * DK + lane * E32, qv);
      load_vec<InT, EV>(reinterpret_cast<const InT*>(p.v) + (bt * p.H + h) * DV + lane * EV, vv);
      g_t = __ldg(p.g + bt * p.H + h);
      beta_t = __ldg(p.beta + bt * p.H + h);
    }
    float nrm[3] = {0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int e = 0; e < E32; ++e) {
      nrm[0] = fmaf(kv[e], kv[e], nrm[0]);
      nrm[1] = fmaf(qv[e], qv[e], nrm[1]);
      nrm[2] = fmaf(kv[e], qv[e], nrm[2]);
    }
    group_allreduce<32, 3>(nrm);
    const float rk = p.l2norm ? rsqrtf(nrm[0] + p.l2_eps) : 1.0f;
    const float rq = p.l2norm ? rsqrtf(nrm[1] + p.l2_eps) : 1.0f;
#pragma unroll
    for (int e = 0; e < E32; ++e) {
      kv[e] *= rk;
      qv[e] *= rq;
    }
    const float kq = nrm[2] * rk * rq;
    const float alpha = expf(g_t);
    const float beta = beta_t;
    const int filled = count < R ? count : R;
    const int pos = count % R;  // ring position of the new update (the oldest when full)

    // decay weights of this warp's entries; entries not yet made weigh 0
    cw = (lane < E && j0 + lane < filled) ? cw * alpha : 0.0f;

    // pass 1: d_j = k_j . k and e_j = k_j . q, interleaved as red[2j], red[2j+1]
    float red[2 * E];
#pragma unroll
    for (int j = 0; j < E; ++j) {
      float kr[E32];
      load_vec<float, E32>(Ks + j * DK + lane * E32, kr);
      float a = 0.0f, c = 0.0f;
#pragma unroll
      for (int e = 0; e < E32; ++e) {
        a = fmaf(kr[e], kv[e], a);
        c = fmaf(kr[e], qv[e], c);
      }
      red[2 * j] = (j0 + j < filled) ? a : 0.0f;
      red[2 * j + 1] = (j0 + j < filled) ? c : 0.0f;
    }
    warp_reduce_scatter<2 * E>(red, lane);
    if constexpr (2 * E >= 32) {
#pragma unroll
      for (int i = 0; i < 2 * E / 32; ++i) my_sums[lane * (2 * E / 32) + i] = red[i];
    } else {
      my_sums[lane >> 1] = red[0];
    }
    __syncwarp();

    // pass 2: this warp's share of the prediction and read-out sums
    float pv[EV], ov[EV];
#pragma unroll
    for (int e = 0; e < EV; ++e) pv[e] = ov[e] = 0.0f;
#pragma unroll
    for (int j = 0; j < E; ++j) {
      const float cj = __shfl_sync(kFull, cw, j);
      float ur[EV];
      load_vec<float, EV>(Us + j * DV + lane * EV, ur);
      const float wp = cj * my_sums[2 * j];
      // the entry at `pos` is replaced when the window is full: it is not
      // part of the window the read-out sees
      const float wo = (filled == R && j0 + j == pos) ? 0.0f : cj * my_sums[2 * j + 1];
      if (j0 + j < filled) {
#pragma unroll
        for (int e = 0; e < EV; ++e) {
          pv[e] = fmaf(wp, ur[e], pv[e]);
          ov[e] = fmaf(wo, ur[e], ov[e]);
        }
      }
    }
    if constexpr (S > 1) {
      // the unit's S partial sums, added in warp order by every warp
      float* mine = part + ((size_t)warp * 2 + (t & 1)) * 2 * DV;
#pragma unroll
      for (int e = 0; e < EV; ++e) {
        mine[lane * EV + e] = pv[e];
        mine[DV + lane * EV + e] = ov[e];
      }
      unit_barrier<S, UPC>(ul);
#pragma unroll
      for (int e = 0; e < EV; ++e) pv[e] = ov[e] = 0.0f;
#pragma unroll
      for (int w2 = 0; w2 < S; ++w2) {
        const float* other = part + ((size_t)(ul * S + w2) * 2 + (t & 1)) * 2 * DV;
#pragma unroll
        for (int e = 0; e < EV; ++e) {
          pv[e] += other[lane * EV + e];
          ov[e] += other[DV + lane * EV + e];
        }
      }
    }
    float dlt[EV];
#pragma unroll
    for (int e = 0; e < EV; ++e) {
      dlt[e] = beta * (vv[e] - pv[e]);
      if (wu == 0)
        store_scalar(out + (bt * p.H + h) * DV + lane * EV + e, p.scale * fmaf(kq, dlt[e], ov[e]));
    }
    // the warp owning ring position `pos` stores the new entry in its slice
    // (for the next token) and in the pool, once it has read its slice
    __syncwarp();
    if (pos >= j0 && pos < j0 + E) {
      const int jl = pos - j0;
#pragma unroll
      for (int e = 0; e < E32; ++e) {
        Ks[jl * DK + lane * E32 + e] = kv[e];
        K[(size_t)pos * DK + lane * E32 + e] = kv[e];
      }
#pragma unroll
      for (int e = 0; e < EV; ++e) {
        Us[jl * DV + lane * EV + e] = dlt[e];
        U[(size_t)pos * DV + lane * EV + e] = dlt[e];
      }
      if (lane == jl) cw = 1.0f;
    }
    ++count;
    __syncwarp();
  }
  // the decay weights and the count, once
  const int filled = count < R ? count : R;
  if (lane < E && j0 + lane < filled) Cw[j0 + lane] = cw;
  if (wu == 0 && lane == 0) *count_p = count;
}

}  // namespace gdn
