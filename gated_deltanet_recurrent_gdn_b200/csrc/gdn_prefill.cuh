// Chunked prefill of the gated delta rule (sm_100a).
//
// A prompt of L tokens is cut into chunks of C = 64 tokens.  Within a chunk
// starting from state S0 (dk x dv), with gamma_i the decay accumulated from
// the chunk start through token i (exp of the running sum of g), the
// token-by-token recurrence is exactly
//
//   A_ij  = beta_i (k_i . k_j) gamma_i / gamma_j             (j < i)
//   Delta = (I + A)^-1 diag(beta) (V - diag(gamma) K S0)      (C x dv)
//         = U - W S0,  U = (I+A)^-1 diag(beta) V,  W = (I+A)^-1 diag(beta gamma) K
//   O     = scale (diag(gamma) Q S0 + P Delta),  P_ij = (q_i . k_j) gamma_i / gamma_j (j <= i)
//   S_end = gamma_C S0 + (K * gamma_C / gamma)^T Delta
//
// (rows of K and Q are the L2-normalised tokens; Delta_i is the delta-rule
// correction of token i).  Everything that does not involve S0 (A, its
// inverse, W, U, P and the decay-scaled Q and K) is independent across
// chunks, so the work splits into two kernels:
//
//   phase A  one CTA per (chunk, head): builds those chunk matrices and
//            writes them to a caller-provided workspace;
//   phase B  one CTA per (sequence, head, 32-column tile of dv): walks the
//            chunks of its sequence in order, carrying its fp32 slice of S
//            in shared memory.  The dv columns of S never interact, so the
//            tiles need no communication.
//
// Both phases compute in fp32 on the CUDA cores.
#pragma once

#include "gdn_kernels.cuh"

namespace gdn {

constexpr int kChunk = 64;
constexpr int kPrefillTile = 32;  // dv columns of S per phase-B CTA

struct PrefillParams {
  const void* q;            // [total][Hk][dk]
  const void* k;            // [total][Hk][dk]
  const void* v;            // [total][H][dv]
  const float* g;           // [total][H]
  const float* beta;        // [total][H]
  float* state;             // [n_slots][H][dv][dk]
  const int32_t* slot_idx;  // [N]
  const int32_t* cu_seqlens;  // [N+1]
  void* out;                // [total][H][dv]
  float* ws;                // [chunk slots][H][ChunkWs::SIZE]
  int N, total, Hk, H, dv, n_slots, group;
  float scale, l2_eps;
  int l2norm, initial_state;
  int* dev_status;
};

// Floats of workspace per (chunk, head).
template <int DK, int DV>
struct ChunkWs {
  static constexpr int W = 0;                          // [C][DK]
  static constexpr int U = W + kChunk * DK;            // [C][DV]
  static constexpr int QG = U + kChunk * DV;           // [C][DK]  gamma_i q_i
  static constexpr int KD = QG + kChunk * DK;          // [C][DK]  k_j gamma_C / gamma_j
  static constexpr int P = KD + kChunk * DK;           // [C][C]
  static constexpr int GL = P + kChunk * kChunk;       // gamma_C
  static constexpr int SIZE = GL + 4;                  // keeps every block 16-byte aligned
};

// A sequence's token range [a, b) is usable when 0 <= a <= b <= total;
// an unusable one owns no chunks and is skipped (and reported) by phase B.
__device__ __forceinline__ long long seq_chunks(int a, int b, int total) {
  return (a < 0 || b < a || b > total) ? 0 : (b - a + kChunk - 1) / kChunk;
}

// Chunks are numbered sequence by sequence, ceil(L/C) per sequence.  Find the
// sequence n, first token t0 and length len of global chunk x (false past the
// last chunk).
__device__ __forceinline__ bool locate_chunk(const int32_t* cu, int N, int total, long long x,
                                             int& n, int& t0, int& len) {
  for (int m = 0; m < N; ++m) {
    const int a = __ldg(cu + m), b = __ldg(cu + m + 1);
    const long long nc = seq_chunks(a, b, total);
    if (x < nc) {
      n = m;
      t0 = a + (int)x * kChunk;
      len = min(kChunk, b - t0);
      return true;
    }
    x -= nc;
  }
  return false;
}

// First global chunk of sequence n.
__device__ __forceinline__ long long first_chunk(const int32_t* cu, int n, int total) {
  long long x = 0;
  for (int m = 0; m < n; ++m) x += seq_chunks(__ldg(cu + m), __ldg(cu + m + 1), total);
  return x;
}

// acc[r][c] += sum_k A(i0+r, k) B(k, j0+c) over k < KD, with
// A(i, k) = A[i * a_i + k * a_k] and B(k, j) = B[k * b_k + j * b_j].
template <int KD, int TM, int TN>
__device__ __forceinline__ void tile_gemm(const float* A, int a_i, int a_k, const float* B,
                                          int b_k, int b_j, int i0, int j0,
                                          float (&acc)[TM][TN]) {
#pragma unroll 4
  for (int kk = 0; kk < KD; ++kk) {
    float a[TM], b[TN];
#pragma unroll
    for (int r = 0; r < TM; ++r) a[r] = A[(i0 + r) * a_i + kk * a_k];
#pragma unroll
    for (int c = 0; c < TN; ++c) b[c] = B[kk * b_k + (j0 + c) * b_j];
#pragma unroll
    for (int r = 0; r < TM; ++r)
#pragma unroll
      for (int c = 0; c < TN; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
  }
}

// Shared-memory floats of phase A.
template <int DK, int DV>
struct PhaseASmem {
  static constexpr int LDK = DK + 1;  // padded rows: row-strided reads hit distinct banks
  static constexpr int LDM = (DK > DV ? DK : DV) + 1;  // q rows, later beta * v rows
  static constexpr int LDC = kChunk + 1;
  static constexpr int KS = 0;                        // [C][LDK] k_hat
  static constexpr int QS = KS + kChunk * LDK;        // [C][LDM] q_hat, later beta v
  static constexpr int AS = QS + kChunk * LDM;        // [C][LDC] A
  static constexpr int TS = AS + kChunk * LDC;        // [C][LDC] (I + A)^-1
  static constexpr int GS = TS + kChunk * LDC;        // [C] running log decay
  static constexpr int BS = GS + kChunk;              // [C] beta
  static constexpr int FLOATS = BS + kChunk;
};

// Phase A: the chunk matrices.  Grid (chunk slots, H); 256 threads.
template <int DK, int DV, typename InT>
__global__ void __launch_bounds__(256) prefill_chunk_kernel(const PrefillParams p) {
  constexpr int C = kChunk;
  constexpr int E = DK / 32;
  using SM = PhaseASmem<DK, DV>;
  using WS = ChunkWs<DK, DV>;
  constexpr int LDK = SM::LDK, LDM = SM::LDM, LDC = SM::LDC;
  extern __shared__ __align__(16) float sm[];
  float* Ks = sm + SM::KS;
  float* Qs = sm + SM::QS;
  float* As = sm + SM::AS;
  float* Ts = sm + SM::TS;
  float* Gs = sm + SM::GS;
  float* Bs = sm + SM::BS;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long x = blockIdx.x;
  const int h = blockIdx.y;
  const int kh = h / p.group;
  int n, t0, len;
  if (!locate_chunk(p.cu_seqlens, p.N, p.total, x, n, t0, len)) return;
  const int s = __ldg(p.slot_idx + n);
  if (s < 0 || s >= p.n_slots) return;  // padding (phase B writes its zeros)
  float* ws = p.ws + ((size_t)x * p.H + h) * WS::SIZE;

  // 1. normalised k and q rows (zero past the chunk), beta and g
  for (int i = warp; i < C; i += 8) {
    float kv[E], qv[E];
    if (i < len) {
      const size_t base = ((size_t)(t0 + i) * p.Hk + kh) * DK + lane * E;
      load_vec<InT, E>(reinterpret_cast<const InT*>(p.k) + base, kv);
      load_vec<InT, E>(reinterpret_cast<const InT*>(p.q) + base, qv);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) kv[e] = qv[e] = 0.0f;
    }
    float red[2] = {0.0f, 0.0f};
#pragma unroll
    for (int e = 0; e < E; ++e) {
      red[0] = fmaf(kv[e], kv[e], red[0]);
      red[1] = fmaf(qv[e], qv[e], red[1]);
    }
    group_allreduce<32, 2>(red);
    const float rk = p.l2norm ? rsqrtf(red[0] + p.l2_eps) : 1.0f;
    const float rq = p.l2norm ? rsqrtf(red[1] + p.l2_eps) : 1.0f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      Ks[i * LDK + lane * E + e] = kv[e] * rk;
      Qs[i * LDM + lane * E + e] = qv[e] * rq;
    }
  }
  if (warp == 0) {
    // inclusive scan of g over the chunk (two tokens per lane)
    float g0 = 0.0f, g1 = 0.0f, b0 = 0.0f, b1 = 0.0f;
    const int i0 = 2 * lane, i1 = 2 * lane + 1;
    if (i0 < len) {
      g0 = __ldg(p.g + (size_t)(t0 + i0) * p.H + h);
      b0 = __ldg(p.beta + (size_t)(t0 + i0) * p.H + h);
    }
    if (i1 < len) {
      g1 = __ldg(p.g + (size_t)(t0 + i1) * p.H + h);
      b1 = __ldg(p.beta + (size_t)(t0 + i1) * p.H + h);
    }
    float run = g0 + g1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_up_sync(kFull, run, off);
      if (lane >= off) run += y;
    }
    Gs[i1] = run;
    Gs[i0] = run - g1;
    Bs[i0] = b0;
    Bs[i1] = b1;
  }
  __syncthreads();

  // 2. A = tril(beta_i (k_i.k_j) gamma_i/gamma_j, -1) and P = tril((q_i.k_j) gamma_i/gamma_j)
  {
    const int i0 = (tid >> 4) * 4, j0 = (tid & 15) * 4;
    float kk[4][4] = {}, qk[4][4] = {};
    tile_gemm<DK, 4, 4>(Ks, LDK, 1, Ks, 1, LDK, i0, j0, kk);
    tile_gemm<DK, 4, 4>(Qs, LDM, 1, Ks, 1, LDK, i0, j0, qk);
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int i = i0 + r, j = j0 + c;
        const float dec = (j <= i) ? __expf(Gs[i] - Gs[j]) : 0.0f;
        As[i * LDC + j] = (j < i) ? Bs[i] * kk[r][c] * dec : 0.0f;
        ws[WS::P + i * C + j] = qk[r][c] * dec;
      }
  }
  __syncthreads();

  // 3. T = (I + A)^-1, column by column: x_i = [i == c] - sum_{c <= j < i} A_ij x_j.
  //    Four lanes per column split the sum; the 64 columns are independent,
  //    so a warp only synchronises with itself.
  //    Every lane walks all C rows (rows above the diagonal are zero), so the
  //    quad shuffles always have the whole warp present.
  {
    const int c = tid >> 2, part = tid & 3;
    for (int i = 0; i < C; ++i) {
      float acc = 0.0f;
      if (i > c)
        for (int j = c + part; j < i; j += 4) acc = fmaf(As[i * LDC + j], Ts[j * LDC + c], acc);
      acc += __shfl_xor_sync(kFull, acc, 1);
      acc += __shfl_xor_sync(kFull, acc, 2);
      if (part == 0) Ts[i * LDC + c] = (i < c) ? 0.0f : ((i == c) ? 1.0f : 0.0f) - acc;
      __syncwarp();
    }
  }
  __syncthreads();

  // 4. decay-scaled q and k, and W = T diag(beta gamma) K
  const float gl = Gs[C - 1];  // padded tokens have g = 0, so this is the last token's
  for (int e = tid; e < C * DK; e += 256) {
    const int i = e / DK, d = e % DK;
    ws[WS::QG + e] = Qs[i * LDM + d] * __expf(Gs[i]);
    ws[WS::KD + e] = Ks[i * LDK + d] * __expf(gl - Gs[i]);
  }
  if (tid == 0) ws[WS::GL] = __expf(gl);
  __syncthreads();
  // scale the rows of K by beta_j gamma_j (in place)
  for (int e = tid; e < C * DK; e += 256) {
    const int j = e / DK, d = e % DK;
    Ks[j * LDK + d] *= Bs[j] * __expf(Gs[j]);
  }
  // v rows (times beta) into the q buffer
  for (int e = tid; e < C * DV / 4; e += 256) {
    const int j = e / (DV / 4), d4 = (e % (DV / 4)) * 4;
    float vv[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (j < len)
      load_vec<InT, 4>(reinterpret_cast<const InT*>(p.v) + ((size_t)(t0 + j) * p.H + h) * DV + d4,
                       vv);
#pragma unroll
    for (int u = 0; u < 4; ++u) Qs[j * LDM + d4 + u] = vv[u] * Bs[j];
  }
  __syncthreads();
  // W = T (diag(beta gamma) K) and U = T (diag(beta) V): 4 rows x (DK/16 or
  // DV/16) columns per thread
  {
    static_assert(DK % 16 == 0 && DV % 16 == 0, "head sizes must be multiples of 16");
    const int i0 = (tid >> 4) * 4;
    {
      const int jb = (tid & 15) * (DK / 16);
      float w[4][DK / 16] = {};
      tile_gemm<C, 4, DK / 16>(Ts, LDC, 1, Ks, LDK, 1, i0, jb, w);
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < DK / 16; ++c) ws[WS::W + (i0 + r) * DK + jb + c] = w[r][c];
    }
    {
      const int jb = (tid & 15) * (DV / 16);
      float u[4][DV / 16] = {};
      tile_gemm<C, 4, DV / 16>(Ts, LDC, 1, Qs, LDM, 1, i0, jb, u);
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < DV / 16; ++c) ws[WS::U + (i0 + r) * DV + jb + c] = u[r][c];
    }
  }
}

// Shared-memory floats of phase B.
template <int DK>
struct PhaseBSmem {
  static constexpr int LDK = DK + 1;
  static constexpr int LDC = kChunk + 1;
  static constexpr int LDT = kPrefillTile + 1;
  static constexpr int SS = 0;                        // [DK][LDT]  S slice (dk x 32)
  static constexpr int WSM = SS + DK * LDT;           // [C][LDK]   W
  static constexpr int QG = WSM + kChunk * LDK;       // [C][LDK]   gamma q
  static constexpr int KD = QG + kChunk * LDK;        // [C][LDK]   k gamma_C / gamma
  static constexpr int PS = KD + kChunk * LDK;        // [C][LDC]   P
  static constexpr int US = PS + kChunk * LDC;        // [C][LDT]   U slice
  static constexpr int DS = US + kChunk * LDT;        // [C][LDT]   Delta slice
  static constexpr int FLOATS = DS + kChunk * LDT;
};

// Phase B: the state through the chunks.  Grid (N, H, dv / 32); 256 threads.
template <int DK, int DV, typename OutT>
__global__ void __launch_bounds__(256) prefill_state_kernel(const PrefillParams p) {
  constexpr int C = kChunk, TL = kPrefillTile;
  using SM = PhaseBSmem<DK>;
  using WS = ChunkWs<DK, DV>;
  constexpr int LDK = SM::LDK, LDC = SM::LDC, LDT = SM::LDT;
  extern __shared__ __align__(16) float sm[];
  float* Ss = sm + SM::SS;
  float* Wm = sm + SM::WSM;
  float* Qg = sm + SM::QG;
  float* Kd = sm + SM::KD;
  float* Ps = sm + SM::PS;
  float* Us = sm + SM::US;
  float* Ds = sm + SM::DS;

  const int tid = threadIdx.x;
  const int n = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * TL;
  const int t0 = __ldg(p.cu_seqlens + n), t1 = __ldg(p.cu_seqlens + n + 1);
  OutT* out = reinterpret_cast<OutT*>(p.out);
  if (t0 < 0 || t1 < t0 || t1 > p.total) {
    if (p.dev_status != nullptr && threadIdx.x == 0) atomicOr(p.dev_status, GDN_STATUS_SEQ_RANGE);
    return;
  }
  const int s = __ldg(p.slot_idx + n);
  if (s < 0 || s >= p.n_slots) {
    if (s != -1 && p.dev_status != nullptr && tid == 0) atomicOr(p.dev_status, GDN_STATUS_SLOT_RANGE);
    for (int e = tid; e < (t1 - t0) * TL; e += 256)
      store_scalar(out + ((size_t)(t0 + e / TL) * p.H + h) * DV + j0 + e % TL, 0.0f);
    return;
  }

  // the state slice: pool rows j0..j0+31 (dk contiguous each) -> Ss[d][c]
  float* pool = p.state + (((size_t)s * p.H + h) * DV + j0) * DK;
  for (int e = tid; e < TL * DK; e += 256) {
    const int c = e / DK, d = e % DK;
    Ss[d * LDT + c] = p.initial_state ? pool[(size_t)c * DK + d] : 0.0f;
  }

  const long long x0 = first_chunk(p.cu_seqlens, n, p.total);
  const int nc = (t1 - t0 + C - 1) / C;
  for (int ch = 0; ch < nc; ++ch) {
    const float* ws = p.ws + ((size_t)(x0 + ch) * p.H + h) * WS::SIZE;
    const int len = min(C, t1 - t0 - ch * C);
    __syncthreads();  // the previous chunk is done with the buffers
    for (int e = tid; e < C * DK / 4; e += 256) {
      const int i = (4 * e) / DK, d = (4 * e) % DK;
      const float4 w = *reinterpret_cast<const float4*>(ws + WS::W + 4 * e);
      const float4 qg = *reinterpret_cast<const float4*>(ws + WS::QG + 4 * e);
      const float4 kd = *reinterpret_cast<const float4*>(ws + WS::KD + 4 * e);
      float* wr = Wm + i * LDK + d;
      float* qr = Qg + i * LDK + d;
      float* kr = Kd + i * LDK + d;
      wr[0] = w.x; wr[1] = w.y; wr[2] = w.z; wr[3] = w.w;
      qr[0] = qg.x; qr[1] = qg.y; qr[2] = qg.z; qr[3] = qg.w;
      kr[0] = kd.x; kr[1] = kd.y; kr[2] = kd.z; kr[3] = kd.w;
    }
    for (int e = tid; e < C * C / 4; e += 256) {
      const int i = (4 * e) / C, j = (4 * e) % C;
      const float4 pv = *reinterpret_cast<const float4*>(ws + WS::P + 4 * e);
      float* pr = Ps + i * LDC + j;
      pr[0] = pv.x; pr[1] = pv.y; pr[2] = pv.z; pr[3] = pv.w;
    }
    for (int e = tid; e < C * TL; e += 256) {
      const int i = e / TL, c = e % TL;
      Us[i * LDT + c] = ws[WS::U + i * DV + j0 + c];
    }
    const float gamma_c = ws[WS::GL];
    __syncthreads();

    // Delta = U - W S and the first half of O (diag(gamma) Q S), 2 x 4 per thread
    const int i0 = (tid >> 3) * 2, c0 = (tid & 7) * 4;
    float ws_[2][4] = {}, qs_[2][4] = {};
    tile_gemm<DK, 2, 4>(Wm, LDK, 1, Ss, LDT, 1, i0, c0, ws_);
    tile_gemm<DK, 2, 4>(Qg, LDK, 1, Ss, LDT, 1, i0, c0, qs_);
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) Ds[(i0 + r) * LDT + c0 + c] = Us[(i0 + r) * LDT + c0 + c] - ws_[r][c];
    __syncthreads();

    // O = scale (diag(gamma) Q S + P Delta) for the chunk's tokens
    tile_gemm<C, 2, 4>(Ps, LDC, 1, Ds, LDT, 1, i0, c0, qs_);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int i = i0 + r;
      if (i < len) {
        OutT* o = out + ((size_t)(t0 + ch * C + i) * p.H + h) * DV + j0 + c0;
#pragma unroll
        for (int c = 0; c < 4; ++c) store_scalar(o + c, p.scale * qs_[r][c]);
      }
    }

    // S <- gamma_C S + Kd^T Delta, DK/32 x 4 per thread
    constexpr int TMS = DK / 32;
    const int d0 = (tid >> 3) * TMS;
    float sn[TMS][4] = {};
    tile_gemm<C, TMS, 4>(Kd, 1, LDK, Ds, LDT, 1, d0, c0, sn);
    __syncthreads();  // every read of the old S is done
#pragma unroll
    for (int r = 0; r < TMS; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float* sp = Ss + (d0 + r) * LDT + c0 + c;
        *sp = fmaf(gamma_c, *sp, sn[r][c]);
      }
  }
  __syncthreads();
  for (int e = tid; e < TL * DK; e += 256) {
    const int c = e / DK, d = e % DK;
    pool[(size_t)c * DK + d] = Ss[d * LDT + c];
  }
}

}  // namespace gdn
