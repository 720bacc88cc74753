// The low-rank sliding window over whole prompts, in chunks (sm_100a).
//
// "GDN tuning limits on Kunlun XPU", section 三.3, runs the low-rank chain
// over a prompt in chunks (and reports that kernel crashing at a prefill of
// 256 concurrent prompts).  The result is defined token by token (the
// low-rank decode step: every token pushes its update (k, delta) into a
// window of the R most recent updates, each keeping the decay accumulated
// since it was made).  Every token's prediction sees the R updates made
// before it, so within a chunk the updates form a banded lower-triangular
// system.  For a chunk of C >= R tokens starting at token a, with the
// window entering it held oldest first (entry e = update a - R + e, weight
// w_e at the chunk start; missing entries weigh 0) and Gamma_t the decay
// from the chunk start through token t:
//
//   KE_te = [e >= t] w_e exp(Gamma_t) (k_t . k_e)      entering entries seen
//   A_ts  = [s < t <= s + R] beta_t exp(Gamma_t - Gamma_s) (k_t . k_s)
//   (I + A) Delta = diag(beta) (V - KE U_entering)
//   QE_te = [e > t] w_e exp(Gamma_t) (q_t . k_e)       after the push
//   PQ_ts = [s <= t < s + R] exp(Gamma_t - Gamma_s) (q_t . k_s)
//   O     = scale (QE U_entering + PQ Delta)
//
// (q, k normalised; t, s, e local to the chunk) and the window leaving the
// chunk is the last R of [entering entries, the chunk's tokens] with their
// weights at the chunk end.  The identity is pinned in numpy against the
// token-by-token definition.
//
// One CTA per (sequence, head), 256 threads, walking its chunks in order on
// the CUDA cores (fp32): the four C x C products of a chunk, the unit lower
// triangular inverse of (I + A) by 16 x 16 blocks, then Delta, the outputs
// and the new window.  Blocks take the prompts longest first.
#pragma once

#include "gdn_lowrank.cuh"
#include "gdn_prefill.cuh"

namespace gdn {

struct LowrankPrefillParams {
  const void* q;            // [total][Hk][dk]
  const void* k;            // [total][Hk][dk]
  const void* v;            // [total][H][dv]
  const float* g;           // [total][H]
  const float* beta;        // [total][H]
  float* win_k;             // [n_slots][H][R][dk]
  float* win_u;             // [n_slots][H][R][dv]
  float* win_c;             // [n_slots][H][R]
  int32_t* win_count;       // [n_slots][H]
  const int32_t* slot_idx;  // [N]
  const int32_t* cu_seqlens;  // [N+1]
  void* out;                // [total][H][dv]
  int N, total, Hk, H, R, n_slots, group;
  float scale, l2_eps;
  int l2norm, initial_window;
  int* dev_status;
};

// Shared-memory floats (C = 64 tokens, windows of up to RM = 64 entries).
template <int DK, int DV>
struct LrpSmem {
  static constexpr int C = kChunk, RM = 64;
  static constexpr int LK = DK + 4, LV = DV + 4;  // rows of the k-like and v-like buffers
  static constexpr int LM = C + 1;                // rows of the C x C and C x RM matrices
  static constexpr int LT = C + 8;                // rows of T^T
  static constexpr int QDS =
      (C * LK > 2 * C * LM ? C * LK : 2 * C * LM) > C * LV ? (C * LK > 2 * C * LM ? C * LK : 2 * C * LM)
                                                           : C * LV;
  static constexpr int KC = 0;                 // [C][LK] normalised k rows of the chunk
  static constexpr int QD = KC + C * LK;       // [C][LK] normalised q rows; then KE and A; then Delta [C][LV]
  static constexpr int KE = QD;                // [C][LM]
  static constexpr int AM = QD + C * LM;       // [C][LM]
  static constexpr int VC = QD + QDS;          // [C][LV] v rows, then the right-hand side
  static constexpr int EK = VC + C * LV;       // [RM][LK] the window's k, oldest first
  static constexpr int EU = EK + RM * LK;      // [RM][LV] its u
  static constexpr int EW = EU + RM * LV;      // [RM] its weights
  static constexpr int QE = EW + RM;           // [C][LM]
  static constexpr int PQ = QE + C * LM;       // [C][LM]
  static constexpr int TT = PQ + C * LM;       // [C][LT] T^T
  static constexpr int YS = TT + C * LT;       // [3][16][17] scratch of the inverse
  static constexpr int GS = YS + 3 * 16 * 17;  // [C] running log decay of the chunk
  static constexpr int BS = GS + C;            // [C] beta
  static constexpr int FLOATS = BS + C;
  static_assert(FLOATS * 4 <= 232448 - 64, "one CTA's shared memory");
};

// An 8 x 8 tile of X Y^T (X, Y row-major with rows of LX, LY floats; D
// columns): thread tile (ti, tj) takes rows 8 r + ti of X and 8 c + tj of Y,
// so the rows a warp reads at once are consecutive (distinct banks).
template <int D, int LX, int LY>
__device__ __forceinline__ void tile_xyt(const float* X, const float* Y, int ti, int tj,
                                         float (&acc)[8][8]) {
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[r][c] = 0.0f;
#pragma unroll 2
  for (int d = 0; d < D; d += 4) {
    float4 x[8], y[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) x[r] = *reinterpret_cast<const float4*>(X + (8 * r + ti) * LX + d);
#pragma unroll
    for (int c = 0; c < 8; ++c) y[c] = *reinterpret_cast<const float4*>(Y + (8 * c + tj) * LY + d);
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        acc[r][c] = fmaf(x[r].x, y[c].x, acc[r][c]);
        acc[r][c] = fmaf(x[r].y, y[c].y, acc[r][c]);
        acc[r][c] = fmaf(x[r].z, y[c].z, acc[r][c]);
        acc[r][c] = fmaf(x[r].w, y[c].w, acc[r][c]);
      }
  }
}

template <int DK, int DV, typename InT, typename OutT>
__global__ void __launch_bounds__(256, 1) lowrank_prefill_kernel(const LowrankPrefillParams p) {
  using SM = LrpSmem<DK, DV>;
  constexpr int C = kChunk, LK = SM::LK, LV = SM::LV, LM = SM::LM, LT = SM::LT;
  static_assert(DK % 32 == 0 && DV % 32 == 0, "head sizes");
  extern __shared__ __align__(128) float lrp_smem[];
  float* sm = lrp_smem;
  float* KC = sm + SM::KC;
  float* QC = sm + SM::QD;
  float* KE = sm + SM::KE;
  float* AM = sm + SM::AM;
  float* DL = sm + SM::QD;  // Delta, once KE and A are consumed
  float* VC = sm + SM::VC;
  float* EK = sm + SM::EK;
  float* EU = sm + SM::EU;
  float* EW = sm + SM::EW;
  float* QE = sm + SM::QE;
  float* PQ = sm + SM::PQ;
  float* Tt = sm + SM::TT;
  float* Ys = sm + SM::YS;
  float* Gs = sm + SM::GS;
  float* Bs = sm + SM::BS;
  __shared__ int pick;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = (int)(blockIdx.x % (unsigned)p.H);
  const int n = longest_first_sequence(p.cu_seqlens, p.N, p.H, p.total, &pick);
  const int t0 = __ldg(p.cu_seqlens + n), t1 = __ldg(p.cu_seqlens + n + 1);
  OutT* out = reinterpret_cast<OutT*>(p.out);
  if (t0 < 0 || t1 < t0 || t1 > p.total) {
    if (p.dev_status != nullptr && tid == 0) atomicOr(p.dev_status, GDN_STATUS_SEQ_RANGE);
    return;
  }
  const int s = __ldg(p.slot_idx + n);
  if (s < 0 || s >= p.n_slots) {
    if (s != -1 && p.dev_status != nullptr && tid == 0) atomicOr(p.dev_status, GDN_STATUS_SLOT_RANGE);
    for (int e = tid; e < (t1 - t0) * DV; e += 256)
      store_scalar(out + ((size_t)(t0 + e / DV) * p.H + h) * DV + e % DV, 0.0f);
    return;
  }
  const int R = p.R;
  const int kh = h / p.group;
  const size_t sh = (size_t)s * p.H + h;
  float* Kp = p.win_k + sh * R * DK;
  float* Up = p.win_u + sh * R * DV;
  float* Cp = p.win_c + sh * R;
  const int count0 = p.initial_window ? *(p.win_count + sh) : 0;

  // the entering window, oldest first in slots R - m .. R - 1 (m = the
  // updates it holds); the other slots, and R .. RM - 1, weigh 0
  {
    const int m = count0 < R ? count0 : R;
    for (int i = tid; i < SM::RM * (DK / 4); i += 256) {
      const int e = i / (DK / 4), d4 = (i % (DK / 4)) * 4;
      float4 x = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      if (e < R && e >= R - m) {
        const int ring = (count0 - R + e) % R;
        x = *reinterpret_cast<const float4*>(Kp + (size_t)ring * DK + d4);
      }
      *reinterpret_cast<float4*>(EK + e * LK + d4) = x;
    }
    for (int i = tid; i < SM::RM * (DV / 4); i += 256) {
      const int e = i / (DV / 4), d4 = (i % (DV / 4)) * 4;
      float4 x = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      if (e < R && e >= R - m) {
        const int ring = (count0 - R + e) % R;
        x = *reinterpret_cast<const float4*>(Up + (size_t)ring * DV + d4);
      }
      *reinterpret_cast<float4*>(EU + e * LV + d4) = x;
    }
    if (tid < SM::RM) EW[tid] = (tid < R && tid >= R - m) ? Cp[(count0 - R + tid) % R] : 0.0f;
  }

  const int nc = (t1 - t0 + C - 1) / C;
  // thread tile of the C x C products: matrix mt, tile (ti, tj)
  const int mt = tid >> 6, tt = tid & 63, ti = tt >> 3, tj = tt & 7;
  // thread tile of the C x dv products: tokens tq + 16 r (r < 4), columns 8 tc .. 8 tc + 7
  const int tq = tid & 15, tc = tid >> 4;
  static_assert(DV <= 128, "16 column blocks of 8 cover dv");
  for (int ch = 0; ch < nc; ++ch) {
    const int a0 = t0 + ch * C;
    const int len = min(C, t1 - a0);
    // 1. normalised k and q rows, v rows (zero past the sequence); g and beta
    {
      const int i = tid >> 2, part = tid & 3;
      constexpr int QK = DK / 4, QV = DV / 4;
      float kv[QK], qv[QK];
      if (i < len) {
        const size_t base = ((size_t)(a0 + i) * p.Hk + kh) * DK + part * QK;
#pragma unroll
        for (int c = 0; c < QK; c += 8) {
          load_vec<InT, 8>(reinterpret_cast<const InT*>(p.k) + base + c, *reinterpret_cast<float(*)[8]>(kv + c));
          load_vec<InT, 8>(reinterpret_cast<const InT*>(p.q) + base + c, *reinterpret_cast<float(*)[8]>(qv + c));
        }
      } else {
#pragma unroll
        for (int c = 0; c < QK; ++c) kv[c] = qv[c] = 0.0f;
      }
      float nk = 0.0f, nq = 0.0f;
#pragma unroll
      for (int c = 0; c < QK; ++c) {
        nk = fmaf(kv[c], kv[c], nk);
        nq = fmaf(qv[c], qv[c], nq);
      }
      nk += __shfl_xor_sync(kFull, nk, 1);
      nq += __shfl_xor_sync(kFull, nq, 1);
      nk += __shfl_xor_sync(kFull, nk, 2);
      nq += __shfl_xor_sync(kFull, nq, 2);
      const float rk = p.l2norm ? rsqrtf(nk + p.l2_eps) : 1.0f;
      const float rq = p.l2norm ? rsqrtf(nq + p.l2_eps) : 1.0f;
#pragma unroll
      for (int c = 0; c < QK; c += 4) {
        *reinterpret_cast<float4*>(KC + i * LK + part * QK + c) =
            make_float4(kv[c] * rk, kv[c + 1] * rk, kv[c + 2] * rk, kv[c + 3] * rk);
        *reinterpret_cast<float4*>(QC + i * LK + part * QK + c) =
            make_float4(qv[c] * rq, qv[c + 1] * rq, qv[c + 2] * rq, qv[c + 3] * rq);
      }
      float vv[QV];
      if (i < len) {
        const size_t base = ((size_t)(a0 + i) * p.H + h) * DV + part * QV;
#pragma unroll
        for (int c = 0; c < QV; c += 8)
          load_vec<InT, 8>(reinterpret_cast<const InT*>(p.v) + base + c, *reinterpret_cast<float(*)[8]>(vv + c));
      } else {
#pragma unroll
        for (int c = 0; c < QV; ++c) vv[c] = 0.0f;
      }
#pragma unroll
      for (int c = 0; c < QV; c += 4)
        *reinterpret_cast<float4*>(VC + i * LV + part * QV + c) =
            make_float4(vv[c], vv[c + 1], vv[c + 2], vv[c + 3]);
    }
    if (warp == 0) {
      // inclusive scan of g over the chunk, two tokens per lane (zero past it)
      const int i0 = 2 * lane, i1 = 2 * lane + 1;
      const float g0 = i0 < len ? __ldg(p.g + (size_t)(a0 + i0) * p.H + h) : 0.0f;
      const float g1 = i1 < len ? __ldg(p.g + (size_t)(a0 + i1) * p.H + h) : 0.0f;
      float run = g0 + g1;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(kFull, run, off);
        if (lane >= off) run += y;
      }
      Gs[i1] = run;
      Gs[i0] = run - g1;
      Bs[i0] = i0 < len ? __ldg(p.beta + (size_t)(a0 + i0) * p.H + h) : 0.0f;
      Bs[i1] = i1 < len ? __ldg(p.beta + (size_t)(a0 + i1) * p.H + h) : 0.0f;
    }
    __syncthreads();

    // 2. the four C x C products with their masks and decays:
    //    mt 0: PQ = q k^T (output band), 1: QE = q k_window^T,
    //    2: KE = k k_window^T (into the q buffer's place: computed after
    //       every q product has read q, see the barrier), 3: A = k k^T (band)
    {
      float acc[8][8];
      if (mt < 2) tile_xyt<DK, LK, LK>(QC, mt == 0 ? KC : EK, ti, tj, acc);
      else tile_xyt<DK, LK, LK>(KC, mt == 2 ? EK : KC, ti, tj, acc);
      __syncthreads();  // every read of q done: KE and A may overwrite it
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int t = 8 * r + ti;
        const float gt = Gs[t];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int x = 8 * c + tj;
          float val;
          if (mt == 0) {  // s = x: s <= t < s + R
            val = (x <= t && t - x < R) ? __expf(gt - Gs[x]) * acc[r][c] : 0.0f;
            PQ[t * LM + x] = val;
          } else if (mt == 1) {  // window entry e = x seen after the push: e > t
            val = (x > t && x < R) ? EW[x] * __expf(gt) * acc[r][c] : 0.0f;
            QE[t * LM + x] = val;
          } else if (mt == 2) {  // window entry e = x seen by the prediction: e >= t
            val = (x >= t && x < R) ? EW[x] * __expf(gt) * acc[r][c] : 0.0f;
            KE[t * LM + x] = val;
          } else {  // s = x: s < t <= s + R
            val = (x < t && t - x <= R) ? Bs[t] * __expf(gt - Gs[x]) * acc[r][c] : 0.0f;
            AM[t * LM + x] = val;
          }
        }
      }
    }
    __syncthreads();

    // 3. T = (I + A)^-1 (ends with a barrier)
    invert_unit_lower64<LM, LT>(AM, Tt, Ys, tid);

    // 4. the right-hand side beta (v - KE U) in place of v; the window's part
    //    of the outputs, QE U, kept in registers
    float o1[4][8];
    {
      float m[4][8];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) m[r][c] = o1[r][c] = 0.0f;
      if (8 * tc < DV) {
        for (int e = 0; e < R; ++e) {
          const float4 u0 = *reinterpret_cast<const float4*>(EU + e * LV + 8 * tc);
          const float4 u1 = *reinterpret_cast<const float4*>(EU + e * LV + 8 * tc + 4);
          const float u[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int t = tq + 16 * r;
            const float ke = KE[t * LM + e], qe = QE[t * LM + e];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              m[r][c] = fmaf(ke, u[c], m[r][c]);
              o1[r][c] = fmaf(qe, u[c], o1[r][c]);
            }
          }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int t = tq + 16 * r;
          float* vr = VC + t * LV + 8 * tc;
#pragma unroll
          for (int c = 0; c < 8; ++c) vr[c] = Bs[t] * (vr[c] - m[r][c]);
        }
      }
    }
    __syncthreads();  // the right-hand side complete; KE and A consumed

    // 5. Delta = T rhs (T lower triangular), where KE and A were
    if (8 * tc < DV) {
      float dl[4][8];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) dl[r][c] = 0.0f;
      for (int x = 0; x < C; ++x) {
        const float4 b0 = *reinterpret_cast<const float4*>(VC + x * LV + 8 * tc);
        const float4 b1 = *reinterpret_cast<const float4*>(VC + x * LV + 8 * tc + 4);
        const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float tv = Tt[x * LT + tq + 16 * r];  // T[t][x]
#pragma unroll
          for (int c = 0; c < 8; ++c) dl[r][c] = fmaf(tv, bv[c], dl[r][c]);
        }
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        float* d = DL + (tq + 16 * r) * LV + 8 * tc;
        *reinterpret_cast<float4*>(d) = make_float4(dl[r][0], dl[r][1], dl[r][2], dl[r][3]);
        *reinterpret_cast<float4*>(d + 4) = make_float4(dl[r][4], dl[r][5], dl[r][6], dl[r][7]);
      }
    }
    __syncthreads();

    // 6. outputs: scale (QE U + PQ Delta)
    if (8 * tc < DV) {
      for (int x = 0; x < C; ++x) {
        const float4 d0 = *reinterpret_cast<const float4*>(DL + x * LV + 8 * tc);
        const float4 d1 = *reinterpret_cast<const float4*>(DL + x * LV + 8 * tc + 4);
        const float dv8[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float pq = PQ[(tq + 16 * r) * LM + x];
#pragma unroll
          for (int c = 0; c < 8; ++c) o1[r][c] = fmaf(pq, dv8[c], o1[r][c]);
        }
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int t = tq + 16 * r;
        if (t < len) {
          OutT* o = out + ((size_t)(a0 + t) * p.H + h) * DV + 8 * tc;
#pragma unroll
          for (int c = 0; c < 8; ++c) store_scalar(o + c, p.scale * o1[r][c]);
        }
      }
    }

    // 7. the window leaving the chunk: the last R of [entering entries, the
    //    chunk's len tokens], with their weights at the chunk end (read
    //    everything first, then write: entries move towards the front)
    {
      const float gl = Gs[C - 1];  // padded tokens have g = 0: the last token's
      constexpr int PK = (SM::RM * DK + 255) / 256, PV = (SM::RM * DV + 255) / 256;
      float kx[PK], ux[PV], wx = 0.0f;
#pragma unroll
      for (int j = 0; j < PK; ++j) {
        const int i = tid + 256 * j, e = i / DK, d = i % DK;
        const int src = e + len;  // index into [entering (R), chunk (len)]
        kx[j] = 0.0f;
        if (e < R) kx[j] = src < R ? EK[src * LK + d] : KC[(src - R) * LK + d];
      }
#pragma unroll
      for (int j = 0; j < PV; ++j) {
        const int i = tid + 256 * j, e = i / DV, d = i % DV;
        const int src = e + len;
        ux[j] = 0.0f;
        if (e < R) ux[j] = src < R ? EU[src * LV + d] : DL[(src - R) * LV + d];
      }
      if (tid < R) {
        const int src = tid + len;
        wx = src < R ? EW[src] * __expf(gl) : __expf(gl - Gs[src - R]);
      }
      __syncthreads();
#pragma unroll
      for (int j = 0; j < PK; ++j) {
        const int i = tid + 256 * j, e = i / DK, d = i % DK;
        if (e < SM::RM) EK[e * LK + d] = kx[j];
      }
#pragma unroll
      for (int j = 0; j < PV; ++j) {
        const int i = tid + 256 * j, e = i / DV, d = i % DV;
        if (e < SM::RM) EU[e * LV + d] = ux[j];
      }
      if (tid < R) EW[tid] = wx;
      __syncthreads();
    }
  }

  // the window back to its ring: update number u lives in position u % R
  const int count = count0 + (t1 - t0);
  const int m = count < R ? count : R;
  for (int i = tid; i < R * DK; i += 256) {
    const int e = i / DK, d = i % DK;
    if (e >= R - m) Kp[(size_t)((count - R + e) % R) * DK + d] = EK[e * LK + d];
  }
  for (int i = tid; i < R * DV; i += 256) {
    const int e = i / DV, d = i % DV;
    if (e >= R - m) Up[(size_t)((count - R + e) % R) * DV + d] = EU[e * LV + d];
  }
  if (tid < R && tid >= R - m) Cp[(count - R + tid) % R] = EW[tid];
  if (tid == 0) *(p.win_count + sh) = count;
}

}  // namespace gdn
