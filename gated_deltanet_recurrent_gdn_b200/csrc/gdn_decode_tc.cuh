// Calls of 2..4 tokens on a 16-bit state pool (bf16 or fp16) with dk = dv =
// 128: the block form of the recurrence (gdn_kernels.cuh) with both of its
// contractions on the 5th-generation tensor cores.
//
// A 16-bit state tile is an exact MMA operand of its own type (kind::f16
// takes bf16 or fp16, the same type for both operands), so the dot products
// of every state row with the call's normalised k and q,
//   X = S0 [k_0 q_0 k_1 q_1 ...]                          (128 x 2T)
// run as one tcgen05.mma pass (M = 128 state rows, K = dk) with the fp32
// vectors split into three parts of the pool's type (x = x1 + x2 + x3, each
// part the rounding of what the previous ones left: about 2^-24 |x| in all
// for bf16; for fp16, whose small parts can fall below its normal range,
// within 2^-25 absolutely, the vectors being of unit length): every part
// product is exact and the accumulation is fp32.  The rank-n update of
// the state after n tokens,
//   S_n = D_{n-1} S0 + Delta,  Delta_ji = sum_{u<n} c_ju k_ui,  c_ju = G(u, n-1) d_ju
// is a second MMA (M = 128 rows, N = 128 columns in two halves, K = 6 part pairs per
// token): with both c and k in three parts, the pairs (a, b) with a + b <= 4
// (counting from 1) leave an error of about 2^-24 of the products, far
// inside the 16-bit storage; for fp16 each row's coefficients are first
// scaled by a power of two into [0.5, 1) (undone exactly in the epilogue),
// so that no part leaves fp16's range.  Each thread owns one state row (TMEM lane r):
// it reads its 2T dot products, runs the token recurrence of its row with
// no shuffles, writes its row's c parts, and after the update MMA forms
// D S0 + Delta for its row and rounds it to the pool's type once, in place in
// the tile.
// The tile comes in and goes back by TMA (two boxes of 64 columns x 128
// rows with the 128-byte swizzle, which is the tensor cores' K-major layout
// and spreads a row's 16-byte chunks over the banks), so neither direction
// takes per-thread memory instructions.  The CUDA cores do about 3
// operations per state element instead of the 8 + 5 of the CUDA-core block
// form.
//
// The grid is one CTA per resident slot (four per SM), each walking the
// (sequence, head) units blockIdx.x, blockIdx.x + gridDim.x, ...: a unit
// never waits for a CTA to be launched or retired, and the mbarriers and the
// tensor memory are set up once per CTA.  A CTA holds 64 TMEM columns: the
// dots take 32, then the update runs as two MMAs of 64 state columns, each
// followed by its half of the epilogue.  (With 128 columns per CTA, measured:
// the fourth CTA of an SM waited in tcgen05.alloc until another released its
// columns, so an SM held about three working CTAs.)
#pragma once

#include <cuda.h>

#include <type_traits>

#include "gdn_prefill_tc.cuh"

namespace gdn {
namespace dtc {

constexpr int R = 128;  // state rows (dv) = threads = TMEM lanes
constexpr int D = 128;  // dk

// Shared memory (bytes, from a 1024-byte aligned base).  The tile is in the
// 128-byte swizzled K-major layout (two regions of 64 columns); the other
// MMA operands are K-major without swizzle (tcb::koff).
constexpr int A0 = 0;                       // S0 tile, then S_n: 2 x [R][64] 16-bit
constexpr int A0_HALF = R * 64 * 2;
constexpr int A0_BYTES = 2 * A0_HALF;
constexpr int U = A0 + A0_BYTES;            // first the dots' B: [32][D] 16-bit,
constexpr int B1_BYTES = 32 * D * 2;        //   then the update's A [R][32] and
constexpr int A2 = U;                       //   B [D][32] 16-bit
constexpr int B2 = U + R * 32 * 2;
constexpr int U_BYTES = 2 * R * 32 * 2;
constexpr int QKP = D + 4;                  // floats per normalised vector (padded: see below)
constexpr int QK = U + U_BYTES;             // normalised k, q: [T][2][QKP] fp32
constexpr int QK_BYTES = kBlockTokens * 2 * QKP * 4;
constexpr int SC = QK + QK_BYTES;           // k.q [T], gram [2][6], tokens' a, beta [2][T]
constexpr int SC_FLOATS = kBlockTokens + 12 + 2 * kBlockTokens;
constexpr int BAR = SC + ((SC_FLOATS * 4 + 15) / 16) * 16;  // 2 mbarriers, TMEM slot, flag
constexpr int BYTES = BAR + 32;
constexpr int ALLOC = BYTES + 1024;         // dynamic shared memory, with the alignment slack
static_assert(B1_BYTES <= U_BYTES, "the dots' operand fits where the update's go");
// 4 CTAs per SM by shared memory at most (4 x 64 TMEM columns)
static_assert(5 * (ALLOC + 1024) > 228 * 1024 && 4 * (ALLOC + 1024) <= 228 * 1024,
              "4 CTAs per SM");
constexpr uint32_t TM_COLS = 64;  // the dots (32 columns), then each half of the update (64)

// Byte offset of 16-byte chunk c (elements 8c .. 8c + 7) of row r in the
// swizzled tile: the chunk's position within its 128-byte row is xor-ed with
// r mod 8 (what the TMA box with the 128-byte swizzle does).
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
  return (uint32_t)((c >> 3) * A0_HALF + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Descriptor of a K-major operand in the 128-byte swizzled layout (8-row
// groups 1024 bytes apart); a K step of 16 elements advances the start by
// 32 bytes within the swizzled rows.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// TMA box of the tile (64 columns from column x, 128 rows from row y) into
// shared memory, completing on `bar`; and back from shared memory.
__device__ __forceinline__ void tma_load_box(const CUtensorMap* map, uint32_t dst, int x, int y,
                                             uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_store_box(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];\n" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(src)
               : "memory");
}

// x rounded to the 16-bit type St, as a float
template <typename St>
__device__ __forceinline__ float round_to(float x);
template <>
__device__ __forceinline__ float round_to<__nv_bfloat16>(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}
template <>
__device__ __forceinline__ float round_to<__half>(float x) {
  return __half2float(__float2half_rn(x));
}

// The three parts of 8 consecutive values in the type St, packed: part 0 is
// their rounding, part n the rounding of what parts 0..n-1 left (each
// subtraction is exact in fp32).
template <typename St>
__device__ __forceinline__ void split3(const float (&x)[8], uint4 (&out)[3]) {
  float rem[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) rem[e] = x[e];
#pragma unroll
  for (int a = 0; a < 3; ++a) {
    uint32_t w[4];
#pragma unroll
    for (int e2 = 0; e2 < 4; ++e2) {
      const float h0 = round_to<St>(rem[2 * e2]), h1 = round_to<St>(rem[2 * e2 + 1]);
      w[e2] = pack2(St(), h0, h1);
      rem[2 * e2] -= h0;
      rem[2 * e2 + 1] -= h1;
    }
    out[a] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Instruction descriptor of kind::f16 with A and B of type St (bf16 or
// fp16), an fp32 accumulator and both operands K-major, for an M x N tile.
template <typename St, int M, int N>
__host__ __device__ constexpr uint32_t idesc16() {
  return std::is_same<St, __half>::value
             ? (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24)
             : idesc_bf16_f32<M, N>();
}

}  // namespace dtc

// `tmap` describes the pool (of type StT) as [n_slots * H * dv] rows of dk =
// 128 elements (256 bytes apart), boxes of 64 x 128 with the 128-byte swizzle.
template <int TT, typename InT, typename OutT, typename StT>
__global__ void __launch_bounds__(128, 4)
    decode_block_tc16_kernel(const StepParams p, const __grid_constant__ CUtensorMap tmap) {
  using namespace dtc;
  using tcb::koff;
  static_assert(TT >= 2 && TT <= kBlockTokens, "block calls take 2..4 tokens");
  static_assert(sizeof(StT) == 2, "16-bit pools");
  extern __shared__ __align__(128) unsigned char dtc_smem[];
  unsigned char* sm = dtc_smem + ((1024u - (smem_u32(dtc_smem) & 1023u)) & 1023u);
  float* qk_s = reinterpret_cast<float*>(sm + QK);
  float* kq_s = reinterpret_cast<float*>(sm + SC);
  float* gram = kq_s + kBlockTokens;  // [2][6]: k_u.k_t, k_u.q_t (u < t)
  float* tok = gram + 12;             // [2][T]: a_t, beta_t
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + BAR);  // the MMAs
  uint64_t* bar_tile = bar + 1;                            // the tile's copy
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 2);
  int* flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int r = threadIdx.x, lane = r & 31, warp = r >> 5;
  OutT* out = reinterpret_cast<OutT*>(p.out);
  const int units = p.B * p.H;

  // Once per CTA: the two mbarriers and the tensor memory.  The CTA then
  // walks the (sequence, head) units blockIdx.x, blockIdx.x + gridDim.x, ...
  // (one CTA per resident slot), so no unit waits for a CTA to be launched
  // or retired; each barrier's completions are counted in ph_*.
  if (r == 0) {
    mbar_init(bar, 1);
    mbar_init(bar_tile, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, TM_COLS);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tm = *tmem_slot;
  uint32_t ph_tile = 0, ph_mma = 0;  // the parity each barrier completes next

  // Waits (bounded) on an mbarrier (the tile's copy or the MMAs); on running
  // out, reports, waits once more so that no copy or product lands in
  // released memory, releases the tensor memory, lets the last stores read
  // the tile and returns false for every thread (the units not yet stored
  // are left as they were).
  auto wait_or_bail = [&](uint64_t* on, uint32_t parity) -> bool {
    if (r == 0) *flag = mbar_wait_bounded(on, parity, kWaitLimitNs) ? 1 : 0;
    __syncthreads();
    if (*flag == 0) {
      if (r == 0) {
        if (p.dev_status != nullptr) atomicOr(p.dev_status, GDN_STATUS_TIMEOUT);
        mbar_wait_bounded(on, parity, kWaitLimitNs);
      }
      tc_fence_before_sync();
      __syncthreads();
      if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tm, TM_COLS);
      }
      if (r == 0) asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory");
      return false;
    }
    mbar_try_wait(on, parity);
    tc_fence_after_sync();
    return true;
  };

  for (int unit = blockIdx.x; unit < units; unit += gridDim.x) {
    const int b = fdiv(unit, p.div_h), h = unit - b * p.H;
    const int kh = fdiv(h, p.div_group);

    const int s = __ldg(p.slot_idx + b);
    if (s < 0 || (p.n_slots > 0 && s >= p.n_slots)) {
      if (s != -1 && p.dev_status != nullptr && r == 0) atomicOr(p.dev_status, GDN_STATUS_SLOT_RANGE);
#pragma unroll
      for (int t = 0; t < TT; ++t) store_scalar(out + (((size_t)b * TT + t) * p.H + h) * R + r, 0.0f);
      continue;
    }
    int n_commit = TT;
    if (p.n_accept != nullptr) {
      n_commit = __ldg(p.n_accept + b);
      if (n_commit < 0 || n_commit > TT) {
        if (p.dev_status != nullptr && r == 0) atomicOr(p.dev_status, GDN_STATUS_ACCEPT_RANGE);
        n_commit = 0;
      }
    }

    // the tile first: two TMA boxes, completing on bar_tile, once the
    // previous unit's stores have read the tile they overwrite
    const int row0 = (s * p.H + h) * R;
    if (r == 0) {
      asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory");
      mbar_arrive_expect_tx(bar_tile, A0_BYTES + kWaitTestExtraTx);
      tma_load_box(&tmap, smem_u32(sm + A0), 0, row0, bar_tile);
      tma_load_box(&tmap, smem_u32(sm + A0 + A0_HALF), 64, row0, bar_tile);
    }
    // then the loads, in the order their results are needed: token `warp`'s k
    // and q, this row's v of every token and token r's gates
    float kv[D / 32], qv[D / 32];
    if (warp < TT) {
      const size_t base = (((size_t)b * TT + warp) * p.Hk + kh) * D;
      load_vec<InT, D / 32>(reinterpret_cast<const InT*>(p.k) + base + lane * (D / 32), kv);
      load_vec<InT, D / 32>(reinterpret_cast<const InT*>(p.q) + base + lane * (D / 32), qv);
    }
    float v_r[TT], g_me = 0.0f, b_me = 0.0f;
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      float v1[1];
      load_vec<InT, 1>(reinterpret_cast<const InT*>(p.v) + (((size_t)b * TT + t) * p.H + h) * R + r, v1);
      v_r[t] = v1[0];
    }
    if (r < TT) {
      g_me = __ldg(p.g + ((size_t)b * TT + r) * p.H + h);
      b_me = __ldg(p.beta + ((size_t)b * TT + r) * p.H + h);
    }
    // into L2: this CTA's next unit (one wave of resident CTAs on)
    if (warp == 3) prefetch_future_inputs<InT>(p, R, D, lane, unit, units);
    if (r == 96) future_tile_prefetch<StT>(p, future_tile_begin(p, unit, units), R, D);
    if (warp < TT)
      normalise_loaded<D>(kv, qv, lane, p.l2_eps, p.l2norm, qk_s + 2 * warp * QKP,
                          qk_s + (2 * warp + 1) * QKP, kq_s + warp);
    __syncthreads();

    // the dots' B operand: row 3 (2t + w) + a holds part a of k_t (w = 0) or
    // q_t (w = 1); rows 6T .. 31 are zero.  Thread r takes 8-element chunk r >> 3
    // of vector r & 7 (2T <= 8 vectors): the eight threads of a shared-memory
    // phase write eight different rows (distinct 16-byte slots of a core
    // matrix) and read eight vectors whose padded pitch puts them in distinct
    // banks.
    {
      const int vec = r & 7, c = r >> 3;
      uint4 pt[3] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
      if (vec < 2 * TT) {
        const float4 x0 = *reinterpret_cast<const float4*>(qk_s + vec * QKP + 8 * c);
        const float4 x1 = *reinterpret_cast<const float4*>(qk_s + vec * QKP + 8 * c + 4);
        const float x8[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        split3<StT>(x8, pt);
      }
#pragma unroll
      for (int a = 0; a < 3; ++a)
        *reinterpret_cast<uint4*>(sm + U + koff(3 * vec + a, 8 * c, D / 8)) = pt[a];
      // rows 24 .. 31 (past every call's 6T <= 24): zero
      *reinterpret_cast<uint4*>(sm + U + koff(24 + vec, 8 * c, D / 8)) = make_uint4(0, 0, 0, 0);
    }
    // the Gram entries of token t = warp: k_u.k_t and k_u.q_t for u < t, in one
    // butterfly (each sum over this lane's elements in order, then the warp)
    if (warp >= 1 && warp < TT) {
      constexpr int E = D / 32;
      const float4 kt = *reinterpret_cast<const float4*>(qk_s + 2 * warp * QKP + lane * E);
      const float4 qt = *reinterpret_cast<const float4*>(qk_s + (2 * warp + 1) * QKP + lane * E);
      float red[2 * (TT - 1)];
#pragma unroll
      for (int u = 0; u < TT - 1; ++u) {
        red[2 * u] = red[2 * u + 1] = 0.0f;
        if (u < warp) {
          const float4 ku = *reinterpret_cast<const float4*>(qk_s + 2 * u * QKP + lane * E);
          const float kuv[4] = {ku.x, ku.y, ku.z, ku.w};
          const float ktv[4] = {kt.x, kt.y, kt.z, kt.w};
          const float qtv[4] = {qt.x, qt.y, qt.z, qt.w};
#pragma unroll
          for (int e = 0; e < E; ++e) {
            red[2 * u] = __fmaf_rn(kuv[e], ktv[e], red[2 * u]);
            red[2 * u + 1] = __fmaf_rn(kuv[e], qtv[e], red[2 * u + 1]);
          }
        }
      }
      group_allreduce<32, 2 * (TT - 1)>(red);
      if (lane < 2 * warp) {
        const int u = lane >> 1, which = lane & 1;
        float x = red[0];
#pragma unroll
        for (int i2 = 1; i2 < 2 * (TT - 1); ++i2)
          if (lane == i2) x = red[i2];
        gram[which * 6 + warp * (warp - 1) / 2 + u] = x;
      }
    }
    if (r < TT) {
      tok[r] = expf(g_me);
      tok[kBlockTokens + r] = b_me;
    }

    fence_proxy_async_smem();  // the B operand's parts, for the MMA's reads
    tc_fence_before_sync();
    if (!wait_or_bail(bar_tile, ph_tile)) return;  // the tile landed
    ph_tile ^= 1;

    // the dots: X (TMEM columns 0..31) = S0 B1^T
    if (r == 0) {
      tc_fence_after_sync();
      constexpr uint32_t id = idesc16<StT, 128, 32>();
      const uint32_t sb = smem_u32(sm);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        tc_mma_bf16(tm, sw128_desc(sb + A0 + (ks >> 2) * A0_HALF + (ks & 3) * 32),
                    tcb::kdesc(sb + U + ks * 256, D * 16), id, ks > 0 ? 1u : 0u);
      tc_commit(bar);
    }
    // meanwhile: the decays D_t = a_0 .. a_t and G(u, t) = a_{u+1} .. a_t
    float al[TT], Dd[TT], G[TT][TT];
#pragma unroll
    for (int t = 0; t < TT; ++t) al[t] = tok[t];
#pragma unroll
    for (int t = 0; t < TT; ++t) Dd[t] = t == 0 ? al[0] : __fmul_rn(Dd[t - 1], al[t]);
#pragma unroll
    for (int u = 0; u < TT; ++u) {
      G[u][u] = 1.0f;
#pragma unroll
      for (int t = u + 1; t < TT; ++t) G[u][t] = __fmul_rn(G[u][t - 1], al[t]);
    }
    if (!wait_or_bail(bar, ph_mma)) return;
    ph_mma ^= 1;

    uint32_t xr[32];
    tcb::tmem_ld32(tm + ((uint32_t)(warp * 32) << 16), xr);
    tcb::tmem_wait_ld(xr);
    // the parts of each dot product, smallest first
    float X[2 * TT];
#pragma unroll
    for (int v = 0; v < 2 * TT; ++v)
      X[v] = __fadd_rn(__fadd_rn(__uint_as_float(xr[3 * v + 2]), __uint_as_float(xr[3 * v + 1])),
                       __uint_as_float(xr[3 * v]));

    // the token recurrence of this row
    float dd[TT];
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      float xk = __fmul_rn(Dd[t], X[2 * t]);
      float xq = __fmul_rn(Dd[t], X[2 * t + 1]);
#pragma unroll
      for (int u = 0; u < t; ++u) {
        xk = __fmaf_rn(__fmul_rn(G[u][t], gram[t * (t - 1) / 2 + u]), dd[u], xk);
        xq = __fmaf_rn(__fmul_rn(G[u][t], gram[6 + t * (t - 1) / 2 + u]), dd[u], xq);
      }
      dd[t] = __fmul_rn(tok[kBlockTokens + t], __fsub_rn(v_r[t], xk));
      const float o = __fmul_rn(p.scale, __fmaf_rn(kq_s[t], dd[t], xq));
      store_scalar(out + (((size_t)b * TT + t) * p.H + h) * R + r, o);
    }
    if (n_commit == 0) {  // a verify-only call: the state stays as it was
      tc_fence_before_sync();
      __syncthreads();  // every read of X done before the next unit's products
      continue;
    }

    // the update's operands.  K index 6u + j pairs part a_j of c_u with part
    // b_j of k_u, (a, b) in (1,1) (1,2) (2,1) (1,3) (3,1) (2,2); K 6n .. 31 zero.
    constexpr int PA[6] = {0, 0, 1, 0, 2, 1}, PB[6] = {0, 1, 0, 2, 0, 1};
    const int n = n_commit;
    float Dn = Dd[0];
#pragma unroll
    for (int t = 1; t < TT; ++t)
      if (t < n) Dn = Dd[t];
    float dscale = 1.0f;  // fp16: 2^e, this row's coefficients were scaled by 2^-e
    {
      // row r of A: this row's c_u = G(u, n-1) d_u in parts
      float cu[TT];
#pragma unroll
      for (int u = 0; u < TT; ++u) {
        float g = 1.0f;
#pragma unroll
        for (int t = u + 1; t < TT; ++t)
          if (t < n) g = G[u][t];
        cu[u] = u < n ? __fmul_rn(g, dd[u]) : 0.0f;
      }
      if constexpr (std::is_same<StT, __half>::value) {
        float mx = 0.0f;
#pragma unroll
        for (int u = 0; u < TT; ++u) mx = fmaxf(mx, fabsf(cu[u]));
        int e = 0;
        frexpf(mx, &e);  // mx in [2^(e-1), 2^e), e = 0 for mx = 0
        dscale = ldexpf(1.0f, e);
#pragma unroll
        for (int u = 0; u < TT; ++u) cu[u] = ldexpf(cu[u], -e);  // exact
      }
      float cpart[TT][3];
#pragma unroll
      for (int u = 0; u < TT; ++u) {
        float x = cu[u];
#pragma unroll
        for (int a = 0; a < 3; ++a) {
          const float hi = round_to<StT>(x);
          cpart[u][a] = hi;
          x -= hi;
        }
      }
      // row r of B: column r of the state, k_u[r] in parts
      float kpart[TT][3];
#pragma unroll
      for (int u = 0; u < TT; ++u) {
        float x = u < n ? qk_s[2 * u * QKP + r] : 0.0f;
#pragma unroll
        for (int a = 0; a < 3; ++a) {
          const float hi = round_to<StT>(x);
          kpart[u][a] = hi;
          x -= hi;
        }
      }
      // 32 K values each (the parts are values of the type: packing them is exact),
      // in four 16-byte chunks
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t wa[4], wb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float av[2], bv[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int k = 8 * c + 2 * i + e;
            av[e] = k < 6 * TT ? cpart[k < 6 * TT ? k / 6 : 0][PA[k % 6]] : 0.0f;
            bv[e] = k < 6 * TT ? kpart[k < 6 * TT ? k / 6 : 0][PB[k % 6]] : 0.0f;
          }
          wa[i] = pack2(StT(), av[0], av[1]);
          wb[i] = pack2(StT(), bv[0], bv[1]);
        }
        *reinterpret_cast<uint4*>(sm + A2 + koff(r, 8 * c, 4)) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
        *reinterpret_cast<uint4*>(sm + B2 + koff(r, 8 * c, 4)) = make_uint4(wb[0], wb[1], wb[2], wb[3]);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();  // every row's parts written; every read of X done

    // Delta = A B^T in two halves of 64 state columns, each in TMEM columns
    // 0..63: the half's update MMA, then its epilogue
    auto update_mma = [&](int half) {
      if (r == 0) {
        tc_fence_after_sync();
        constexpr uint32_t id = idesc16<StT, 128, 64>();
        const uint32_t sb = smem_u32(sm);
        // B's rows 64 half .. : eight 8-row groups of 512 bytes each
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
          tc_mma_bf16(tm, tcb::kdesc(sb + A2 + ks * 256, 4 * 128),
                      tcb::kdesc(sb + B2 + half * 8 * 512 + ks * 256, 4 * 128), id,
                      ks > 0 ? 1u : 0u);
        tc_commit(bar);
      }
    };
    update_mma(0);
    // meanwhile: this row of S0, packed, into registers
    uint4 s0[D / 8];
#pragma unroll
    for (int c = 0; c < D / 8; ++c) s0[c] = *reinterpret_cast<const uint4*>(sm + A0 + sw_off(r, c));

    // S_n = D_{n-1} S0 + Delta, rounded once, in place in the tile: columns
    // 0..63 first, stored by TMA while columns 64..127 are formed
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      if (!wait_or_bail(bar, ph_mma)) return;  // (half 0) also: every thread has read its S0 row
      ph_mma ^= 1;
#pragma unroll
      for (int qt = 2 * half; qt < 2 * half + 2; ++qt) {  // 32 columns at a time
        uint32_t dr[32];
        tcb::tmem_ld32(tm + ((uint32_t)(warp * 32) << 16) + 32 * (qt - 2 * half), dr);
        tcb::tmem_wait_ld(dr);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 w = s0[4 * qt + c];
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
          uint32_t o4[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float x0, x1;
            unpack2(StT(), ws[i], x0, x1);
            float d0 = __uint_as_float(dr[8 * c + 2 * i]), d1 = __uint_as_float(dr[8 * c + 2 * i + 1]);
            if constexpr (std::is_same<StT, __half>::value) {
              d0 = __fmul_rn(d0, dscale);  // a power of two: exact
              d1 = __fmul_rn(d1, dscale);
            }
            const float y0 = __fmaf_rn(Dn, x0, d0);
            const float y1 = __fmaf_rn(Dn, x1, d1);
            o4[i] = pack2(StT(), y0, y1);
          }
          *reinterpret_cast<uint4*>(sm + A0 + sw_off(r, 4 * qt + c)) =
              make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
      }
      fence_proxy_async_smem();  // this row's half, for the TMA store's reads
      tc_fence_before_sync();
      __syncthreads();  // every row's half written; every TMEM read of the half done
      if (r == 0) tma_store_box(&tmap, smem_u32(sm + A0 + half * A0_HALF), 64 * half, row0);
      if (half == 0) update_mma(1);
    }
    if (r == 0) asm volatile("cp.async.bulk.commit_group;\n" ::: "memory");
  }
  // the tensor memory back; the tile's shared memory stays until the last
  // unit's stores have read it
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tm, TM_COLS);
  }
  if (r == 0) asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory");
}

}  // namespace gdn
