// Phase B of the chunked prefill on the 5th-generation tensor cores
// (sm_100a tcgen05), for bf16 inputs and dk = dv = 128.
//
// Phase A leaves only T = (I + A)^-1 per (chunk, head) in the workspace.
// This kernel, one CTA per (sequence, head), walks the sequence's chunks and
// forms everything else from the raw bf16 rows of k, q and v.  With rk_i,
// rq_i the inverse norms, G_i the running log decay from the chunk start,
// gamma_i = exp(G_i) and S the dk x dv state at the chunk start, the chunk
// identity of the recurrence (see gdn_prefill.cuh) reads
//
//   Y = K_raw S,  Z = Q_raw S                                  (C x dv)
//   R_ij  = beta_i v_ij - beta_i gamma_i rk_i Y_ij
//   Delta = T R
//   P_ij  = rq_i (q_i . k_j) rk_j exp(G_i - G_j)  for j <= i, else 0
//   O     = scale (diag(gamma rq) Z + P Delta)
//   S    <- gamma_C S + K_raw^T Delta',  Delta'_ij = exp(G_C - G_i) rk_i Delta_ij
//
// Every product runs as tcgen05.mma with dv = 128 as the M of the tile (TMEM
// lane j = state column j), i.e. on the transposes: Y^T = S^T K_raw^T,
// Delta^T = R^T T^T, O^T = Delta^T P^T, S^T += Delta'^T K_raw.  S^T (the
// pool's own [dv][dk] layout) is kept in fp32 in tensor memory as the
// accumulator of the state update.  The raw k and q rows are exact in bf16;
// every fp32 operand is split into bf16 parts, x = x1 + x2 + x3 with each
// part the rounding of what the previous ones left (to about 2^-27 |x|), and
// a product keeps the part products whose error terms stay below fp32
// rounding:
//   K_raw S, S^T K_raw     S in 3 parts               (3 MMA passes)
//   T R                    both in 3 parts, the 6 part pairs (a, b) with
//                          a + b <= 4                  (6 passes)
//   K_raw^T Delta'         Delta' in 3 parts           (3 passes)
//   P Delta (outputs only) both in 2 parts, pairs (1,1) (1,2) (2,1): about
//                          2^-17 relative, far inside the output tolerance
// q . k is one bf16 pass (exact products, fp32 accumulation).
//
// Per chunk: stage 1 (Y, Z and the Gram q k^T) -> R^T parts on the CUDA
// cores -> stage 2 (Delta; P's parts are formed meanwhile) -> Delta parts ->
// stage 3 (O and the state update) -> outputs and the next chunk's S^T parts.
// The next chunk's k/q rows (double-buffered), v rows and T are loaded while
// this one computes.
#pragma once

#include "gdn_prefill.cuh"

namespace gdn {
namespace tcb {

constexpr int C = kChunk;  // tokens per chunk
constexpr int D = 128;     // dk = dv

// Shared memory (bytes).  Operands of the MMAs are K-major without swizzle:
// core matrices of 8 rows x 16 bytes; LBO = 128 bytes between core matrices
// adjacent in K, SBO = (K / 8) x 128 bytes between groups of 8 rows.
constexpr int KQ_BYTES = 2 * C * D * 2;          // [k; q] rows of a chunk, [128][128] bf16
constexpr int KQ0 = 0;                            // two buffers
constexpr int VS = KQ0 + 2 * KQ_BYTES;            // v rows [C][D] bf16, row-major
constexpr int T32 = VS + C * D * 2;               // T [C][C] fp32 in 8 x 8 blocks
constexpr int TP = T32 + C * C * 4;               // T in 3 bf16 parts, [C][C] K-major
constexpr int X = TP + 3 * C * C * 2;             // S^T parts, or the chunk's parts:
constexpr int SP_PART = D * D * 2;                //   S^T [D][D] bf16 x 3
constexpr int RP_PART = D * C * 2;                //   [D][C] bf16 (R^T, Delta^T, Delta'^T)
constexpr int RP = X;                             //   R^T x 3, then Delta'^T x 3
constexpr int DP = RP + 3 * RP_PART;              //   Delta^T x 2
constexpr int PP_PART = C * C * 2;                //   [C][C] bf16
constexpr int PP = DP + 2 * RP_PART;              //   P x 2
constexpr int SC = X + 3 * SP_PART;               // per-token scalars (floats)
constexpr int NSC = 7;                            // RK RQ GS BT CY CZ CD, C each
constexpr int BAR = SC + NSC * C * 4;             // mbarriers and small words
constexpr int BYTES = BAR + 64;
static_assert(PP + 2 * PP_PART <= SC, "the chunk's parts fit where the S^T parts were");
static_assert(BYTES <= 232448, "the shared memory of one CTA");

// Tensor memory columns (fp32 accumulators; 128 lanes = the state columns)
constexpr uint32_t TM_S = 0;     // S^T, the state (128)
constexpr uint32_t TM_YZ = 128;  // Y^T (64) and Z^T (64)
constexpr uint32_t TM_GR = 256;  // [k; q] k^T (64); lanes 64..127 hold q . k
constexpr uint32_t TM_DL = 320;  // Delta^T (64)
constexpr uint32_t TM_OP = 384;  // (P Delta)^T (64)
constexpr uint32_t TM_COLS = 512;

// Byte offset of element (r, c) in a K-major operand with `kc` 8-element
// chunks per row.
__device__ __forceinline__ uint32_t koff(int r, int c, int kc) {
  return (uint32_t)((r >> 3) * kc * 128 + (c >> 3) * 128 + (r & 7) * 16 + (c & 7) * 2);
}

// The NP bf16 parts of 8 consecutive values: part 0 is their rounding to
// bf16, part n the rounding of what parts 0..n-1 left (each subtraction is
// exact in fp32).
template <int NP>
__device__ __forceinline__ void split_parts(const float (&x)[8], uint4 (&out)[NP]) {
  float r[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) r[e] = x[e];
#pragma unroll
  for (int pt = 0; pt < NP; ++pt) {
    uint32_t w[4];
#pragma unroll
    for (int e2 = 0; e2 < 4; ++e2) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(r[2 * e2], r[2 * e2 + 1]);
      w[e2] = *reinterpret_cast<const uint32_t*>(&h);
      r[2 * e2] -= __low2float(h);
      r[2 * e2 + 1] -= __high2float(h);
    }
    out[pt] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// 16 bytes global -> shared, asynchronously; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;\n" ::: "memory");
}

// 32 consecutive TMEM columns of this thread's lane, without waiting.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// Wait for this thread's TMEM loads; naming the registers keeps every use
// of them after the wait.
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;\n"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
        "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
        "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
        "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
        "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
}
// Keeps the uses of a second array of loaded registers after an earlier wait.
__device__ __forceinline__ void tmem_after_wait(uint32_t (&r)[32]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                 "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}
// 32 consecutive TMEM columns of this thread's lane from registers.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}

__device__ __forceinline__ uint64_t kdesc(uint32_t addr, uint32_t sbo) {
  return smem_desc_kmajor(addr, 128, sbo);
}

}  // namespace tcb

// Phase B on tcgen05.  Grid N * H, 256 threads (8 warps), one CTA per SM
// (all 512 TMEM columns, 218 KB of shared memory).  Thread (warp w, lane l)
// owns TMEM lane / state column j = 32 (w % 4) + l and the half w / 4 of
// the columns of every per-chunk tile it reads (tokens 32 (w / 4) ..).
template <typename OutT>
__global__ void __launch_bounds__(256, 1) prefill_state_tc_kernel(const PrefillParams p) {
  using namespace tcb;
  extern __shared__ __align__(128) unsigned char tcb_smem[];
  unsigned char* sm = tcb_smem;
  float* RK = reinterpret_cast<float*>(sm + SC);  // 1 / |k_i|
  float* RQ = RK + C;                             // 1 / |q_i|
  float* GS = RQ + C;                             // running log decay G_i
  float* BT = GS + C;                             // beta_i (0 past the chunk)
  float* CY = BT + C;                             // beta_i gamma_i rk_i
  float* CZ = CY + C;                             // gamma_i rq_i
  float* CD = CZ + C;                             // exp(G_C - G_i) rk_i
  uint64_t* barT = reinterpret_cast<uint64_t*>(sm + BAR);  // T landed
  uint64_t* barM = barT + 1;                                // MMA stages
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(barM + 1);
  int* flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* pick = flag + 1;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = (int)(blockIdx.x % (unsigned)p.H);
  const int n = phase_b_sequence(p, pick);
  const int t0 = __ldg(p.cu_seqlens + n), t1 = __ldg(p.cu_seqlens + n + 1);
  OutT* out = reinterpret_cast<OutT*>(p.out);
  if (t0 < 0 || t1 < t0 || t1 > p.total) {
    if (p.dev_status != nullptr && tid == 0) atomicOr(p.dev_status, GDN_STATUS_SEQ_RANGE);
    return;
  }
  const int s = __ldg(p.slot_idx + n);
  if (s < 0 || s >= p.n_slots) {
    if (s != -1 && p.dev_status != nullptr && tid == 0) atomicOr(p.dev_status, GDN_STATUS_SLOT_RANGE);
    for (int e = tid; e < (t1 - t0) * D; e += 256)
      store_scalar(out + ((size_t)(t0 + e / D) * p.H + h) * D + e % D, 0.0f);
    return;
  }

  const int kh = h / p.group;
  const long long x0 = first_chunk(p.cu_seqlens, n, p.total);
  const int nc = (t1 - t0 + C - 1) / C;
  const float* ws0 = p.ws + ((size_t)x0 * p.H + h) * kTcbWsFloats;
  const size_t chunk_stride = (size_t)p.H * kTcbWsFloats;
  const __nv_bfloat16* kin = reinterpret_cast<const __nv_bfloat16*>(p.k);
  const __nv_bfloat16* qin = reinterpret_cast<const __nv_bfloat16*>(p.q);
  const __nv_bfloat16* vin = reinterpret_cast<const __nv_bfloat16*>(p.v);

  const int jrow = (warp & 3) * 32 + lane;  // TMEM lane: state column j
  const int hc = warp >> 2;                  // which half of a tile's columns
  const uint32_t sbase = smem_u32(sm);

  // the chunk loaders (zeros past the sequence, so every operand is finite)
  auto load_kq = [&](int ch, int buf) {
    const int len = min(C, t1 - t0 - ch * C);
    unsigned char* dst = sm + KQ0 + buf * KQ_BYTES;
    for (int e = tid; e < 2 * C * (D / 8); e += 256) {
      const int r = e >> 4, c = e & 15, i = r & (C - 1);
      const bool ok = i < len;
      const __nv_bfloat16* src = (r < C ? kin : qin) +
                                 (ok ? ((size_t)(t0 + ch * C + i) * p.Hk + kh) * D + 8 * c : 0);
      cp_async16(dst + koff(r, 8 * c, D / 8), src, ok ? 16 : 0);
    }
  };
  auto load_v = [&](int ch) {
    const int len = min(C, t1 - t0 - ch * C);
    for (int e = tid; e < C * (D / 8); e += 256) {
      const int i = e >> 4, c = e & 15;
      const bool ok = i < len;
      const __nv_bfloat16* src = vin + (ok ? ((size_t)(t0 + ch * C + i) * p.H + h) * D + 8 * c : 0);
      cp_async16(sm + VS + i * (D * 2) + c * 16, src, ok ? 16 : 0);
    }
  };
  auto load_t = [&](int ch) {  // one thread
    mbar_arrive_expect_tx(barT, C * C * 4);
    bulk_copy_g2s(sm + T32, ws0 + (size_t)ch * chunk_stride, C * C * 4, barT);
  };
  // T copies issued and waited for (thread 0's count; a copy still in
  // flight when the kernel gives up is waited for before it returns)
  int t_issued = 0, t_waited = 0;
  // g and beta of a chunk: warp 4, two tokens per lane (zero past the sequence)
  float gn0 = 0.0f, gn1 = 0.0f, bn0 = 0.0f, bn1 = 0.0f;
  auto load_gb = [&](int ch) {
    const int len = min(C, t1 - t0 - ch * C);
    const int i0 = 2 * lane, i1 = 2 * lane + 1;
    const size_t base = (size_t)(t0 + ch * C) * p.H + h;
    gn0 = i0 < len ? __ldg(p.g + base + (size_t)i0 * p.H) : 0.0f;
    gn1 = i1 < len ? __ldg(p.g + base + (size_t)i1 * p.H) : 0.0f;
    bn0 = i0 < len ? __ldg(p.beta + base + (size_t)i0 * p.H) : 0.0f;
    bn1 = i1 < len ? __ldg(p.beta + base + (size_t)i1 * p.H) : 0.0f;
  };

  if (warp == 0) tmem_alloc(tmem_slot, TM_COLS);
  if (tid == 0) {
    mbar_init(barT, 1);
    mbar_init(barM, 1);
    fence_mbar_init();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tm = *tmem_slot;
  const uint32_t lane_tm = tm + ((uint32_t)((warp & 3) * 32) << 16);

  if (nc > 0) {
    load_kq(0, 0);
    load_v(0);
    if (tid == 0) {
      load_t(0);
      t_issued = 1;
    }
    if (warp == 4) load_gb(0);
  }

  // the state: pool row j (dk contiguous) is row j of S^T; this thread takes
  // its 64 columns d = 64 hc .. into TMEM and, as 3 bf16 parts, into the
  // operand of stage 1
  float* pool = p.state + ((size_t)s * p.H + h) * D * D;
  {
    uint32_t v[2][32];
    const float4* src = reinterpret_cast<const float4*>(pool + (size_t)jrow * D + 64 * hc);
#pragma unroll
    for (int q4 = 0; q4 < 16; ++q4) {
      const float4 f = p.initial_state ? src[q4] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      v[q4 >> 3][(q4 & 7) * 4 + 0] = __float_as_uint(f.x);
      v[q4 >> 3][(q4 & 7) * 4 + 1] = __float_as_uint(f.y);
      v[q4 >> 3][(q4 & 7) * 4 + 2] = __float_as_uint(f.z);
      v[q4 >> 3][(q4 & 7) * 4 + 3] = __float_as_uint(f.w);
    }
    tmem_st32(lane_tm + TM_S + 64 * hc, v[0]);
    tmem_st32(lane_tm + TM_S + 64 * hc + 32, v[1]);
#pragma unroll
    for (int c8 = 0; c8 < 8; ++c8) {
      float x8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) x8[e] = __uint_as_float(v[c8 >> 2][(c8 & 3) * 8 + e]);
      uint4 pt[3];
      split_parts<3>(x8, pt);
#pragma unroll
      for (int a = 0; a < 3; ++a)
        *reinterpret_cast<uint4*>(sm + X + a * SP_PART + koff(jrow, 64 * hc + 8 * c8, D / 8)) = pt[a];
    }
    tmem_wait_st();
  }

  // Waits on a barrier with a bound; on running out, reports, waits once more
  // (bounded) so that no copy or product lands in released memory, releases
  // the tensor memory and returns false for every thread.
  uint32_t mma_parity = 0;
  auto wait_or_bail = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (tid == 0) *flag = mbar_wait_bounded(bar, parity, kWaitLimitNs) ? 1 : 0;
    __syncthreads();
    const bool ok = *flag != 0;
    if (!ok) {
      if (tid == 0) {
        if (p.dev_status != nullptr) atomicOr(p.dev_status, GDN_STATUS_TIMEOUT);
        mbar_wait_bounded(bar, parity, kWaitLimitNs);
        if (bar != barT && t_issued > t_waited)
          mbar_wait_bounded(barT, (uint32_t)(t_waited & 1), kWaitLimitNs);
      }
      cp_async_wait_all();
      tc_fence_before_sync();
      __syncthreads();
      if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tm, TM_COLS);
      }
      return false;
    }
    mbar_try_wait(bar, parity);  // completed: this thread acquires the result
    tc_fence_after_sync();
    return true;
  };

  for (int ch = 0; ch < nc; ++ch) {
    const int buf = ch & 1;
    const int len = min(C, t1 - t0 - ch * C);
    const uint32_t kq = sbase + KQ0 + buf * KQ_BYTES;
    // 1. this chunk's rows (and, on its barrier, T) in shared memory
    cp_async_wait_all();
    fence_proxy_async_smem();
    tc_fence_before_sync();
    if (!wait_or_bail(barT, ch & 1)) return;
    ++t_waited;

    // stage 1: Y^T, Z^T = S^T [K; Q]^T and the Gram [k; q] k^T
    if (tid == 0) {
      constexpr uint32_t id128 = idesc_bf16_f32<128, 128>();
      constexpr uint32_t id64 = idesc_bf16_f32<128, 64>();
#pragma unroll
      for (int a = 0; a < 3; ++a)
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          tc_mma_bf16(tm + TM_YZ, kdesc(sbase + X + a * SP_PART + ks * 256, D * 16),
                      kdesc(kq + ks * 256, D * 16), id128, (a | ks) != 0 ? 1u : 0u);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        tc_mma_bf16(tm + TM_GR, kdesc(kq + ks * 256, D * 16), kdesc(kq + ks * 256, D * 16), id64,
                    ks != 0 ? 1u : 0u);
      tc_commit(barM);
    }
    // the next chunk's k and q into the other buffer (its last reader, the
    // previous chunk's state update, has completed)
    if (ch + 1 < nc) load_kq(ch + 1, buf ^ 1);

    // 2. norms of the 128 rows; the decay scan; T in 3 parts
    if (tid < 2 * C) {
      const unsigned char* row = sm + KQ0 + buf * KQ_BYTES;
      float ss = 0.0f;
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        float x8[8];
        load_vec<__nv_bfloat16, 8>(
            reinterpret_cast<const __nv_bfloat16*>(row + koff(tid, 8 * c, D / 8)), x8);
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(x8[e], x8[e], ss);
      }
      const float r = p.l2norm ? rsqrtf(ss + p.l2_eps) : 1.0f;
      if (tid < C) RK[tid] = r;
      else RQ[tid - C] = r;
    } else if (warp == 4) {
      // inclusive scan of g over the chunk, as phase A takes it
      const int i0 = 2 * lane, i1 = 2 * lane + 1;
      float run = gn0 + gn1;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(kFull, run, off);
        if (lane >= off) run += y;
      }
      GS[i1] = run;
      GS[i0] = run - gn1;
      BT[i0] = bn0;
      BT[i1] = bn1;
      if (ch + 1 < nc) load_gb(ch + 1);
    }
    for (int task = tid; task < C * (C / 8); task += 256) {
      const int il = task & 7, c8 = (task >> 3) & 7, ib = task >> 6;
      const float4* src =
          reinterpret_cast<const float4*>(sm + T32) + ((ib * (C / 8) + c8) * 64 + il * 8) / 4;
      const float4 a0 = src[0], a1 = src[1];
      const float x8[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      uint4 pt[3];
      split_parts<3>(x8, pt);
#pragma unroll
      for (int a = 0; a < 3; ++a)
        *reinterpret_cast<uint4*>(sm + TP + a * PP_PART + koff(8 * ib + il, 8 * c8, C / 8)) = pt[a];
    }
    fence_proxy_async_smem();  // T's parts, for stage 2; T32's reads before its next copy
    __syncthreads();
    if (tid < C) {
      const int i = tid;
      const float gi = GS[i], gl = GS[C - 1];  // padded tokens have g = 0
      const float e = __expf(gi);
      CY[i] = BT[i] * e * RK[i];
      CZ[i] = e * RQ[i];
      CD[i] = __expf(gl - gi) * RK[i];
    }
    if (tid == 0 && ch + 1 < nc) {
      load_t(ch + 1);
      ++t_issued;
    }
    if (!wait_or_bail(barM, mma_parity)) return;  // stage 1 done (its barrier also publishes C*)
    mma_parity ^= 1;

    // 3. R^T in 3 parts (columns: tokens 32 hc ..) and Z^T scaled (kept for
    //    the outputs)
    float zs[32];
    {
      uint32_t y[32], z[32];
      tmem_ld32(lane_tm + TM_YZ + 32 * hc, y);
      tmem_ld32(lane_tm + TM_YZ + C + 32 * hc, z);
      tmem_wait_ld(y);
      tmem_after_wait(z);
      const __nv_bfloat16* vcol = reinterpret_cast<const __nv_bfloat16*>(sm + VS) + jrow;
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        float r8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int c = 8 * c8 + e, i = 32 * hc + c;
          const float vij = __bfloat162float(vcol[i * D]);
          r8[e] = i < len ? fmaf(BT[i], vij, -CY[i] * __uint_as_float(y[c])) : 0.0f;
          zs[c] = CZ[i] * __uint_as_float(z[c]);
        }
        uint4 pt[3];
        split_parts<3>(r8, pt);
#pragma unroll
        for (int a = 0; a < 3; ++a)
          *reinterpret_cast<uint4*>(sm + RP + a * RP_PART + koff(jrow, 32 * hc + 8 * c8, C / 8)) =
              pt[a];
      }
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();  // R^T ready; v consumed
    tc_fence_after_sync();

    // stage 2: Delta^T = R^T T^T (6 part pairs)
    if (tid == 0) {
      constexpr uint32_t id64 = idesc_bf16_f32<128, 64>();
      constexpr int PA[6] = {0, 0, 1, 0, 1, 2}, PB[6] = {0, 1, 0, 2, 1, 0};
#pragma unroll
      for (int pr = 0; pr < 6; ++pr)
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
          tc_mma_bf16(tm + TM_DL, kdesc(sbase + RP + PA[pr] * RP_PART + ks * 256, C * 16),
                      kdesc(sbase + TP + PB[pr] * PP_PART + ks * 256, C * 16), id64,
                      (pr | ks) != 0 ? 1u : 0u);
      tc_commit(barM);
    }
    if (ch + 1 < nc) load_v(ch + 1);
    // meanwhile: P in 2 parts from lanes 64..127 of the Gram (q rows), for
    // stage 3 (stage 2 reads neither the Gram's columns nor P's buffer)
    if (jrow >= C) {
      const int i = jrow - C;
      uint32_t gr[32];
      tmem_ld32(lane_tm + TM_GR + 32 * hc, gr);
      tmem_wait_ld(gr);
      const float ri = RQ[i], gi = GS[i];
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        float p8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j = 32 * hc + 8 * c8 + e;
          const float dec = (j <= i && i < len) ? __expf(gi - GS[j]) : 0.0f;
          p8[e] = (ri * __uint_as_float(gr[8 * c8 + e]) * RK[j]) * dec;
        }
        uint4 pt[2];
        split_parts<2>(p8, pt);
#pragma unroll
        for (int a = 0; a < 2; ++a)
          *reinterpret_cast<uint4*>(sm + PP + a * PP_PART + koff(i, 32 * hc + 8 * c8, C / 8)) =
              pt[a];
      }
    }
    // and S^T <- gamma_C S^T in tensor memory (stage 3 accumulates onto it)
    {
      const float gam = __expf(GS[C - 1]);
      uint32_t a[32], b[32];
      tmem_ld32(lane_tm + TM_S + 64 * hc, a);
      tmem_ld32(lane_tm + TM_S + 64 * hc + 32, b);
      tmem_wait_ld(a);
      tmem_after_wait(b);
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        a[c] = __float_as_uint(gam * __uint_as_float(a[c]));
        b[c] = __float_as_uint(gam * __uint_as_float(b[c]));
      }
      tmem_st32(lane_tm + TM_S + 64 * hc, a);
      tmem_st32(lane_tm + TM_S + 64 * hc + 32, b);
      tmem_wait_st();
    }
    tc_fence_before_sync();
    if (!wait_or_bail(barM, mma_parity)) return;  // stage 2 done
    mma_parity ^= 1;

    // 4. Delta^T in 2 parts (for the outputs) and Delta'^T in 3 parts (for
    //    the state), the latter where R^T was
    {
      uint32_t dl[32];
      tmem_ld32(lane_tm + TM_DL + 32 * hc, dl);
      tmem_wait_ld(dl);
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        float d8[8], e8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int i = 32 * hc + 8 * c8 + e;
          d8[e] = __uint_as_float(dl[8 * c8 + e]);
          e8[e] = CD[i] * d8[e];
        }
        uint4 pd[2], pe[3];
        split_parts<2>(d8, pd);
        split_parts<3>(e8, pe);
        const uint32_t o = koff(jrow, 32 * hc + 8 * c8, C / 8);
#pragma unroll
        for (int a = 0; a < 2; ++a) *reinterpret_cast<uint4*>(sm + DP + a * RP_PART + o) = pd[a];
#pragma unroll
        for (int a = 0; a < 3; ++a) *reinterpret_cast<uint4*>(sm + RP + a * RP_PART + o) = pe[a];
      }
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();

    // stage 3: (P Delta)^T = Delta^T P^T and S^T += Delta'^T K_raw (K_raw
    // read MN-major from the k rows: LBO = 2 KB between 8-token groups along
    // K, SBO = 128 bytes between 8-element pieces of d along N)
    if (tid == 0) {
      constexpr uint32_t id64 = idesc_bf16_f32<128, 64>();
      constexpr uint32_t id128mn = idesc_bf16_f32<128, 128>() | (1u << 16);
      constexpr int PA[3] = {0, 0, 1}, PB[3] = {0, 1, 0};
#pragma unroll
      for (int pr = 0; pr < 3; ++pr)
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
          tc_mma_bf16(tm + TM_OP, kdesc(sbase + DP + PA[pr] * RP_PART + ks * 256, C * 16),
                      kdesc(sbase + PP + PB[pr] * PP_PART + ks * 256, C * 16), id64,
                      (pr | ks) != 0 ? 1u : 0u);
#pragma unroll
      for (int a = 0; a < 3; ++a)
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
          tc_mma_bf16(tm + TM_S, kdesc(sbase + RP + a * RP_PART + ks * 256, C * 16),
                      smem_desc_kmajor(kq + ks * 2 * (D * 16), D * 16, 128), id128mn, 1u);
      tc_commit(barM);
    }
    if (!wait_or_bail(barM, mma_parity)) return;  // stage 3 done
    mma_parity ^= 1;

    // 5. outputs of the chunk's tokens; the next chunk's S^T parts
    {
      uint32_t op[32];
      tmem_ld32(lane_tm + TM_OP + 32 * hc, op);
      tmem_wait_ld(op);
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const int i = 32 * hc + c;
        if (i < len)
          store_scalar(out + ((size_t)(t0 + ch * C + i) * p.H + h) * D + jrow,
                       p.scale * (zs[c] + __uint_as_float(op[c])));
      }
    }
    if (ch + 1 < nc) {
      uint32_t a[32], b[32];
      tmem_ld32(lane_tm + TM_S + 64 * hc, a);
      tmem_ld32(lane_tm + TM_S + 64 * hc + 32, b);
      tmem_wait_ld(a);
      tmem_after_wait(b);
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        float x8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          x8[e] = __uint_as_float(c8 < 4 ? a[8 * c8 + e] : b[8 * (c8 - 4) + e]);
        uint4 pt[3];
        split_parts<3>(x8, pt);
#pragma unroll
        for (int q = 0; q < 3; ++q)
          *reinterpret_cast<uint4*>(sm + X + q * SP_PART + koff(jrow, 64 * hc + 8 * c8, D / 8)) =
              pt[q];
      }
      fence_proxy_async_smem();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
  }

  // the final state back to the pool: row j of S^T is pool row j
  {
    uint32_t a[32], b[32];
    tmem_ld32(lane_tm + TM_S + 64 * hc, a);
    tmem_ld32(lane_tm + TM_S + 64 * hc + 32, b);
    tmem_wait_ld(a);
    tmem_after_wait(b);
    float4* dst = reinterpret_cast<float4*>(pool + (size_t)jrow * D + 64 * hc);
#pragma unroll
    for (int q4 = 0; q4 < 8; ++q4) {
      dst[q4] = make_float4(__uint_as_float(a[4 * q4]), __uint_as_float(a[4 * q4 + 1]),
                            __uint_as_float(a[4 * q4 + 2]), __uint_as_float(a[4 * q4 + 3]));
      dst[8 + q4] = make_float4(__uint_as_float(b[4 * q4]), __uint_as_float(b[4 * q4 + 1]),
                                __uint_as_float(b[4 * q4 + 2]), __uint_as_float(b[4 * q4 + 3]));
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tm, TM_COLS);
  }
}

}  // namespace gdn
