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
//   phase B  one CTA per (sequence, head): walks the chunks of its sequence
//            in order, carrying the fp32 state in shared memory; each
//            chunk's matrices arrive with one bulk copy, and the next
//            chunk's are requested into L2 while this one is computed.
//
// The products run on the tensor cores.  With bf16 inputs the products of
// phase A run on the 5th-generation tensor cores (tcgen05, accumulators in
// tensor memory): the Gram products K K^T and Q K^T on the raw rows, and
// with dk = dv = 128 also W and U, with T split in three bf16 parts.  The
// other products use warp-level mma.sync with tf32 operands split in hi and
// lo parts for fp32 accuracy.  The triangular solve and the element-wise
// work stay on the CUDA cores.
#pragma once

#include <type_traits>

#include "gdn_kernels.cuh"

namespace gdn {

constexpr int kChunk = 64;

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

// Floats of workspace per (chunk, head), laid out as phase B reads them (it
// copies the whole block into shared memory at once): W, diag(gamma) Q and
// P transposed, so that the tensor-core fragments of phase B are column
// reads.  Rows are padded by 8 floats, which puts the 4 x 8 lanes of a
// fragment load in 32 distinct banks.
template <int DK, int DV>
struct ChunkWs {
  static constexpr int LW = kChunk + 8;                // rows of WT, QGT, PT
  static constexpr int LKD = DK + 8;                   // rows of KD
  static constexpr int LU = DV + 8;                    // rows of U
  static constexpr int WT = 0;                         // [DK][LW]  W^T
  static constexpr int U = WT + DK * LW;               // [C][LU]
  static constexpr int QGT = U + kChunk * LU;          // [DK][LW]  (gamma_i q_i)^T
  static constexpr int KD = QGT + DK * LW;             // [C][LKD]  k_j gamma_C / gamma_j
  static constexpr int PT = KD + kChunk * LKD;         // [C][LW]   P^T: PT[j][i] = P_ij
  static constexpr int GL = PT + kChunk * LW;          // gamma_C
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

// ---------------------------------------------------------------------------
// warp-level tensor-core products, fp32-accurate (3xTF32)
//
// mma.sync m16n8k8 with tf32 operands and fp32 accumulation.  Each fp32
// operand x is split into hi = tf32(x) and lo = tf32(x - hi) (x - hi is exact
// in fp32), and a product takes three MMAs, lo.hi + hi.lo + hi.hi: the
// dropped lo.lo term and the rounding of lo leave a relative error near
// 2^-21, the accuracy of an fp32 product.  Fragments (g = lane / 4,
// t = lane % 4): A (16 x 8) holds (g, t), (g+8, t), (g, t+4), (g+8, t+4);
// B (8 x 8) holds (k=t, n=g), (k=t+4, n=g); C holds (g, 2t), (g, 2t+1),
// (g+8, 2t), (g+8, 2t+1).

__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  hi = to_tf32(x);
  lo = to_tf32(x - __uint_as_float(hi));
}
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4],
                                         const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
__device__ __forceinline__ void mma_3xtf32(float (&d)[4], const uint32_t (&ahi)[4],
                                           const uint32_t (&alo)[4], const uint32_t (&bhi)[2],
                                           const uint32_t (&blo)[2]) {
  mma_tf32(d, alo, bhi);
  mma_tf32(d, ahi, blo);
  mma_tf32(d, ahi, bhi);
}
// A fragment of the 16 x 8 block at (m0, k0) of a matrix stored k-major:
// element (m, k) at A[k * lda + m].
__device__ __forceinline__ void load_a_split(const float* A, int lda, int m0, int k0, int g,
                                             int t, uint32_t (&hi)[4], uint32_t (&lo)[4]) {
  split_tf32(A[(k0 + t) * lda + m0 + g], hi[0], lo[0]);
  split_tf32(A[(k0 + t) * lda + m0 + g + 8], hi[1], lo[1]);
  split_tf32(A[(k0 + t + 4) * lda + m0 + g], hi[2], lo[2]);
  split_tf32(A[(k0 + t + 4) * lda + m0 + g + 8], hi[3], lo[3]);
}
// The same fragment of a matrix stored m-major: element (m, k) at A[m * lda + k].
__device__ __forceinline__ void load_a_split_rows(const float* A, int lda, int m0, int k0, int g,
                                                  int t, uint32_t (&hi)[4], uint32_t (&lo)[4]) {
  split_tf32(A[(m0 + g) * lda + k0 + t], hi[0], lo[0]);
  split_tf32(A[(m0 + g + 8) * lda + k0 + t], hi[1], lo[1]);
  split_tf32(A[(m0 + g) * lda + k0 + t + 4], hi[2], lo[2]);
  split_tf32(A[(m0 + g + 8) * lda + k0 + t + 4], hi[3], lo[3]);
}
// B fragment of the 8 x 8 block at (k0, n0) of a matrix stored n-major:
// element (k, n) at B[n * ldb + k].
__device__ __forceinline__ void load_b_split_cols(const float* B, int ldb, int k0, int n0, int g,
                                                  int t, uint32_t (&hi)[2], uint32_t (&lo)[2]) {
  split_tf32(B[(n0 + g) * ldb + k0 + t], hi[0], lo[0]);
  split_tf32(B[(n0 + g) * ldb + k0 + t + 4], hi[1], lo[1]);
}
// B fragment of the 8 x 8 block at (k0, n0) of a matrix stored row-major
// (k rows): element (k, n) at B[k * ldb + n].
__device__ __forceinline__ void load_b_split(const float* B, int ldb, int k0, int n0, int g,
                                             int t, uint32_t (&hi)[2], uint32_t (&lo)[2]) {
  split_tf32(B[(k0 + t) * ldb + n0 + g], hi[0], lo[0]);
  split_tf32(B[(k0 + t + 4) * ldb + n0 + g], hi[1], lo[1]);
}

// ---------------------------------------------------------------------------
// 5th-generation tensor cores (tcgen05).  One thread issues an MMA whose
// operands are matrices in shared memory, described by 64-bit descriptors;
// the fp32 accumulator lives in tensor memory (TMEM: 128 lanes x columns of
// 32 bits per SM), and the warps read it back with tcgen05.ld, warp w
// reaching lanes 32 (w % 4) .. 32 (w % 4) + 31.

// Allocate `cols` TMEM columns (a power of two >= 32) and write their base
// address to shared memory; the calling warp executes it as a whole.  The
// permit is released at once, so CTAs that arrive later can allocate too.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                   smem_u32(dst)),
               "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(cols)
               : "memory");
}
// Order tcgen05 operations against the CTA barrier between them.
__device__ __forceinline__ void tc_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
// Descriptor of a K-major operand without swizzle: core matrices of 8 rows x
// 16 bytes (128 contiguous bytes), `lbo` bytes between core matrices adjacent
// in K and `sbo` bytes between adjacent groups of 8 rows.
__device__ __forceinline__ uint64_t smem_desc_kmajor(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | ((uint64_t)1 << 46);
}
// Instruction descriptor of kind::f16 with bf16 A and B, an fp32 accumulator
// and both operands K-major, for an M x N tile.
template <int M, int N>
__host__ __device__ constexpr uint32_t idesc_bf16_f32() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}
// D (TMEM) = A B^T (+ D when `accumulate`), K = 16.
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}
// Arrive on `bar` once every MMA this thread issued before has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
          smem_u32(bar))
      : "memory");
}
// 32 consecutive columns of this thread's TMEM lane.  The wait names the
// destination registers, so no use of them can be scheduled before it.
__device__ __forceinline__ void tmem_load32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
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
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;\n"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
        "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
        "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
        "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
        "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}

// Field values of the descriptor of an MN-major operand without swizzle, as
// phase A lays it out (8-element pieces contiguous in M, 8 K-rows of a piece
// 16 bytes apart): LBO = bytes between groups of 8 rows adjacent in K, SBO =
// bytes between the pieces adjacent in M.  (For a K-major operand LBO is
// likewise the step along K, between core matrices adjacent in K.)  A probe
// on B200 matched fp64 with this reading and not with the fields swapped.
#ifndef GDN_MN_LBO
#define GDN_MN_LBO 2048
#define GDN_MN_SBO 128
#endif

// Shared-memory floats of phase A.  K and Q are held row-major ([token][d],
// rows of LDQ = 4 mod 32 floats): the C x C products read them as the
// m-major A and n-major B operand with the 4 x 8 lanes of a fragment load in
// 32 distinct banks, and a warp storing or reading a row touches 32 distinct
// banks.  T = (I + A)^-1 is held transposed (row c = column c of T), which is
// the k-major operand of W = T (beta gamma K) and U = T (beta V); those two
// right-hand sides are row-major with rows of LDR = 8 mod 32 floats, the
// stride at which a k-row B fragment load is conflict free.  The two large
// buffers are reused once their first contents are consumed.  TCB (bf16
// inputs, dk = dv = 128, whose phase B runs on tcgen05) only solves for T:
// it needs no fp32 rows and has no such buffers.
template <int DK, int DV, bool TCB = false>
struct PhaseASmem {
  static constexpr int LDT = kChunk + 8;  // rows of T^T
  static constexpr int LDC = kChunk + 1;  // rows of A
  static constexpr int LDQ = DK + 4;      // rows of K and Q
  static constexpr int MX = DK > DV ? DK : DV;
  static constexpr int LDR = MX + 8;      // rows of beta gamma K and beta V
  static constexpr int BUF =
      TCB ? 0 : ((kChunk * LDQ > kChunk * LDR) ? kChunk * LDQ : kChunk * LDR);
  static constexpr int B1 = 0;               // K [C][LDQ], later beta V [C][LDR]
  static constexpr int B2 = B1 + BUF;        // Q [C][LDQ], later beta gamma K [C][LDR]
  static constexpr int AS = B2 + BUF;        // [C][LDC] A
  static constexpr int TT = AS + kChunk * LDC;  // [C][LDT] T^T
  static constexpr int GS = TT + kChunk * LDT;  // [C] running log decay
  static constexpr int BS = GS + kChunk;        // [C] beta
  static constexpr int EG = BS + kChunk;        // [C] gamma_i = exp(G_i)
  static constexpr int EK = EG + kChunk;        // [C] gamma_C / gamma_i
  static constexpr int EB = EK + kChunk;        // [C] beta_i gamma_i
  static constexpr int YS = EB + kChunk;        // [3][16][17] block products of the solve
  static constexpr int RK = YS + 3 * 16 * 17;   // [C] 1 / |k_i|
  static constexpr int RQ = RK + kChunk;        // [C] 1 / |q_i|
  static constexpr int FLOATS = RQ + kChunk;
  // bf16 inputs: the raw k and q rows as the operand [k; q] (2C rows) of the
  // tcgen05 Gram product, laid out [2C / 8][DK / 8][8 rows][8 elements]: a
  // core matrix is 8 consecutive rows of one 8-element chunk (LBO = 128 bytes
  // between chunks, SBO = DK x 16 bytes between row groups); the k rows are
  // the first half.  It overlays A and T^T, which are written only after the
  // Gram product has completed.
  static constexpr int CB_SBO = DK * 16;
  static constexpr int CB_BYTES = (2 * kChunk / 8) * CB_SBO;
  static constexpr int CB = AS;
  static_assert(CB_BYTES <= (GS - AS) * 4, "the tensor-core copy fits where it is placed");
};

// Workspace floats per (chunk, head) when phase B runs on tcgen05: T alone,
// in 8 x 8 blocks ([C/8][C/8][8][8], element (i, m) of block (i/8, m/8) at
// (i%8)*8 + m%8), so that phase B reads 8 consecutive m of one row i as 32
// contiguous bytes and a quarter warp reads 8 rows of one block at once.
constexpr int kTcbWsFloats = kChunk * kChunk;
__host__ __device__ constexpr int tcb_t_index(int i, int m) {
  return (((i >> 3) * (kChunk / 8) + (m >> 3)) << 6) + ((i & 7) << 3) + (m & 7);
}

// T = (I + A)^-1 for a strictly lower triangular 64 x 64 A (rows of LDC
// floats; entries on and above the diagonal are not read), into T^T (row c
// of Tt = column c of T, rows of LDT floats), by 16 x 16 blocks.  The four
// diagonal blocks are inverted at once by forward substitution (x_i =
// [i == c] - sum_{c <= j < i} A_ij x_j within the block; four lanes per
// column, a warp only synchronises with itself); then the blocks below the
// diagonal follow, one block-diagonal at a time:
//   T_IJ = -T_II sum_{J <= K < I} A_IK T_KJ.
// All 256 threads of the CTA call it; Ys is 3 x 16 x 17 floats of scratch.
// It ends with a CTA barrier.
template <int LDC, int LDT>
__device__ __forceinline__ void invert_unit_lower64(const float* As, float* Tt, float* Ys,
                                                    int tid) {
  {
    const int b = tid >> 6, cc = (tid & 63) >> 2, part = tid & 3;
    const int c = 16 * b + cc;
    float* tc = Tt + c * LDT;
    for (int i = part; i < 16 * b; i += 4) tc[i] = 0.0f;  // rows above the block
    for (int ii = 0; ii < 16; ++ii) {
      const int i = 16 * b + ii;
      float acc = 0.0f;
      if (i > c)
        for (int j = c + part; j < i; j += 4) acc = fmaf(As[i * LDC + j], tc[j], acc);
      acc += __shfl_xor_sync(kFull, acc, 1);
      acc += __shfl_xor_sync(kFull, acc, 2);
      if (part == 0) tc[i] = (i < c) ? 0.0f : ((i == c) ? 1.0f : 0.0f) - acc;
      __syncwarp();
    }
  }
  __syncthreads();
  {
    // element (r, q) of a 16 x 16 block; the 16 lanes of a half warp take 16
    // rows r, so that their reads of A and their stores of T^T are distinct banks
    const int r = tid & 15, q = tid >> 4;
    for (int lvl = 1; lvl < 4; ++lvl) {
      const int nt = 4 - lvl;  // blocks (I, J) = (J + lvl, J), J < nt
      for (int J = 0; J < nt; ++J) {
        const int I = J + lvl;
        float y = 0.0f;
        const float* arow = As + (16 * I + r) * LDC;
        const float* tcol = Tt + (16 * J + q) * LDT;
        for (int k = 16 * J; k < 16 * I; ++k) y = fmaf(arow[k], tcol[k], y);
        Ys[(J * 16 + r) * 17 + q] = y;
      }
      __syncthreads();
      for (int J = 0; J < nt; ++J) {
        const int I = J + lvl;
        float x = 0.0f;
#pragma unroll
        for (int m = 0; m < 16; ++m)
          x = fmaf(Tt[(16 * I + m) * LDT + 16 * I + r], Ys[(J * 16 + m) * 17 + q], x);
        Tt[(16 * J + q) * LDT + 16 * I + r] = -x;
      }
      __syncthreads();
    }
  }
}

// Phase A: the chunk matrices.  Grid (chunk slots, H); 256 threads.
template <int DK, int DV, typename InT>
__global__ void __launch_bounds__(256) prefill_chunk_kernel(const PrefillParams p) {
  constexpr int C = kChunk;
  // bf16 inputs take K K^T and Q K^T on the 5th-generation tensor cores
  constexpr bool TC = std::is_same<InT, __nv_bfloat16>::value;
  // and with dk = dv = 128 the rest of the chunk's products belong to phase
  // B (on tcgen05): this phase only solves for T
  constexpr bool TCB = TC && DK == 128 && DV == 128;
  using SM = PhaseASmem<DK, DV, TCB>;
  using WS = ChunkWs<DK, DV>;
  constexpr int LDT = SM::LDT, LDC = SM::LDC, LDR = SM::LDR, LDQ = SM::LDQ;
  static_assert(DK % 16 == 0 && DV % 16 == 0, "head sizes must be multiples of 16");
  extern __shared__ __align__(128) float sm[];
  float* Ks = sm + SM::B1;  // K, then beta V (absent with TCB)
  float* Qs = sm + SM::B2;  // Q, then beta gamma K (absent with TCB)
  float* As = sm + SM::AS;
  float* Tt = sm + SM::TT;
  float* Gs = sm + SM::GS;
  float* Bs = sm + SM::BS;
  float* Eg = sm + SM::EG;
  float* Ek = sm + SM::EK;
  float* Eb = sm + SM::EB;
  float* Ys = sm + SM::YS;
  float* Rk = sm + SM::RK;
  float* Rq = sm + SM::RQ;
  // the 2C x C fp32 Gram tile
  constexpr uint32_t kTmemCols = kChunk;
  __shared__ uint64_t mma_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int mma_done;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long x = blockIdx.x;
  const int h = blockIdx.y;
  const int kh = h / p.group;
  int n, t0, len;
  if (!locate_chunk(p.cu_seqlens, p.N, p.total, x, n, t0, len)) return;
  const int s = __ldg(p.slot_idx + n);
  if (s < 0 || s >= p.n_slots) return;  // padding (phase B writes its zeros)
  float* ws = p.ws + ((size_t)x * p.H + h) * (TCB ? kTcbWsFloats : WS::SIZE);

  if constexpr (TC) {
    if (warp == 0) tmem_alloc(&tmem_base, kTmemCols);
    if (tid == 0) {
      mbar_init(&mma_bar, 1);
      fence_mbar_init();
    }
  }

  // 1. normalised k and q rows (zero past the chunk); beta and g.  Warp w
  //    takes tokens 8w .. 8w + 7; lane (cl, rl) = (lane / 8, lane % 8) holds
  //    token 8w + rl and its 8-element chunks cl, cl + 4, ...: the 4 lanes of
  //    a token read 64 contiguous bytes per load, its norm is a 2-level
  //    butterfly, and the 8 lanes of a quarter warp write 8 consecutive rows
  //    (distinct banks) of the fp32 buffers and of the tensor-core copy.
  {
    constexpr int NCH = DK / 8;   // 8-element chunks per row
    constexpr int CPL = NCH / 4;  // chunks per lane
    static_assert(NCH % 4 == 0, "4 lanes per token");
    const int rl = lane & 7, cl = lane >> 3;
    const int i = warp * 8 + rl;
    float kv[CPL][8], qv[CPL][8];
    if (i < len) {
      const size_t base = ((size_t)(t0 + i) * p.Hk + kh) * DK;
#pragma unroll
      for (int j = 0; j < CPL; ++j) {
        load_vec<InT, 8>(reinterpret_cast<const InT*>(p.k) + base + 8 * (cl + 4 * j), kv[j]);
        load_vec<InT, 8>(reinterpret_cast<const InT*>(p.q) + base + 8 * (cl + 4 * j), qv[j]);
      }
    } else {
#pragma unroll
      for (int j = 0; j < CPL; ++j)
#pragma unroll
        for (int e = 0; e < 8; ++e) kv[j][e] = qv[j][e] = 0.0f;
    }
    float red[2] = {0.0f, 0.0f};
#pragma unroll
    for (int j = 0; j < CPL; ++j)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        red[0] = fmaf(kv[j][e], kv[j][e], red[0]);
        red[1] = fmaf(qv[j][e], qv[j][e], red[1]);
      }
#pragma unroll
    for (int off = 8; off < 32; off <<= 1) {
      red[0] += __shfl_xor_sync(kFull, red[0], off);
      red[1] += __shfl_xor_sync(kFull, red[1], off);
    }
    const float rk = p.l2norm ? rsqrtf(red[0] + p.l2_eps) : 1.0f;
    const float rq = p.l2norm ? rsqrtf(red[1] + p.l2_eps) : 1.0f;
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
      const int d = 8 * (cl + 4 * j);
      if constexpr (!TCB) {
#pragma unroll
        for (int h4 = 0; h4 < 2; ++h4) {
          *reinterpret_cast<float4*>(Ks + i * LDQ + d + 4 * h4) =
              make_float4(kv[j][4 * h4] * rk, kv[j][4 * h4 + 1] * rk, kv[j][4 * h4 + 2] * rk,
                          kv[j][4 * h4 + 3] * rk);
          *reinterpret_cast<float4*>(Qs + i * LDQ + d + 4 * h4) =
              make_float4(qv[j][4 * h4] * rq, qv[j][4 * h4 + 1] * rq, qv[j][4 * h4 + 2] * rq,
                          qv[j][4 * h4 + 3] * rq);
        }
      }
      if constexpr (TC) {
        // the raw values again as bf16 (exact: they came from bf16)
        unsigned char* cb = reinterpret_cast<unsigned char*>(sm + SM::CB) + (d / 8) * 128;
        uint4 kw, qw;
        kw.x = pack2(__nv_bfloat16(), kv[j][0], kv[j][1]); kw.y = pack2(__nv_bfloat16(), kv[j][2], kv[j][3]);
        kw.z = pack2(__nv_bfloat16(), kv[j][4], kv[j][5]); kw.w = pack2(__nv_bfloat16(), kv[j][6], kv[j][7]);
        qw.x = pack2(__nv_bfloat16(), qv[j][0], qv[j][1]); qw.y = pack2(__nv_bfloat16(), qv[j][2], qv[j][3]);
        qw.z = pack2(__nv_bfloat16(), qv[j][4], qv[j][5]); qw.w = pack2(__nv_bfloat16(), qv[j][6], qv[j][7]);
        *reinterpret_cast<uint4*>(cb + (i / 8) * SM::CB_SBO + (i % 8) * 16) = kw;
        *reinterpret_cast<uint4*>(cb + ((C + i) / 8) * SM::CB_SBO + (i % 8) * 16) = qw;
      }
    }
    if (cl == 0) {
      Rk[i] = rk;
      Rq[i] = rq;
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
    // per-token decay factors (padded tokens have g = 0: the last lane's
    // running sum is the last token's)
    const float gl = __shfl_sync(kFull, run, 31);
    const float e0 = __expf(run - g1), e1 = __expf(run);
    Eg[i0] = e0;
    Eg[i1] = e1;
    Ek[i0] = __expf(gl - (run - g1));
    Ek[i1] = __expf(gl - run);
    Eb[i0] = b0 * e0;
    Eb[i1] = b1 * e1;
  }
  if constexpr (TC) {
    fence_proxy_async_smem();  // the tensor-core copy, for the MMA's reads
    tc_fence_before_sync();
  }
  __syncthreads();
  if constexpr (TC) tc_fence_after_sync();

  // 3. decay-scaled q (transposed) and k (row-major), gamma_C.  For the
  //    transposed store a warp takes 8 tokens x 4 elements: 32 distinct banks
  //    in the row-major Q, four full 32-byte sectors of the workspace.
  const float gl = Gs[C - 1];  // padded tokens have g = 0, so this is the last token's
  auto write_decayed_qk = [&]() {
    for (int e = tid; e < C * DK; e += 256) {
      const int i = ((e >> 5) % (C / 8)) * 8 + (e & 7);
      const int d = (e / (4 * C)) * 4 + ((e >> 3) & 3);
      ws[WS::QGT + d * WS::LW + i] = Qs[i * LDQ + d] * Eg[i];
    }
    for (int e = tid; e < C * DK; e += 256) {
      const int i = e / DK, d = e % DK;
      ws[WS::KD + i * WS::LKD + d] = Ks[i * LDQ + d] * Ek[i];
    }
    if (tid == 0) ws[WS::GL] = __expf(gl);
  };

  // 2. A = tril(beta_i (k_i.k_j) gamma_i/gamma_j, -1) and P = tril((q_i.k_j) gamma_i/gamma_j)
  if constexpr (TC) {
    // bf16 inputs: the Gram tile [k; q] k^T (2C x C) of the raw rows on the
    // 5th-generation tensor cores, issued by one thread (bf16 products are
    // exact in fp32; fp32 accumulation).  The norms and the decays are applied
    // as the tile is read back from TMEM; step 3 runs meanwhile.
    const uint32_t tmem = tmem_base;
    if (tid == 0) {
      const uint32_t cb = smem_u32(sm + SM::CB);
      constexpr uint32_t idesc = idesc_bf16_f32<2 * C, C>();
#pragma unroll
      for (int ks = 0; ks < DK / 16; ++ks) {
        const uint64_t d = smem_desc_kmajor(cb + ks * 256, 128, SM::CB_SBO);
        tc_mma_bf16(tmem, d, d, idesc, ks > 0 ? 1u : 0u);
      }
      tc_commit(&mma_bar);
    }
    if constexpr (!TCB) write_decayed_qk();
    if (tid == 0) mma_done = mbar_wait_bounded(&mma_bar, 0, kWaitLimitNs) ? 1 : 0;
    __syncthreads();
    if (!mma_done) {
      // the product did not complete: report it, give it one more bounded
      // wait, release the tensor memory and leave the chunk unfinished
      if (tid == 0) {
        if (p.dev_status != nullptr) atomicOr(p.dev_status, GDN_STATUS_TIMEOUT);
        mbar_wait_bounded(&mma_bar, 0, kWaitLimitNs);
      }
      tc_fence_before_sync();
      __syncthreads();
      if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
      }
      return;
    }
    mbar_try_wait(&mma_bar, 0);  // completed: every thread acquires the result
    tc_fence_after_sync();
    {
      // warp w reads TMEM lanes 32 (w % 4) .. (rows of [k; q]) and tokens
      // j = 32 (w / 4) .. 32 (w / 4) + 31
      const int row = (warp & 3) * 32 + lane;
      const int c0 = (warp >> 2) * 32;
      float gv[32];
      tmem_load32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)c0, gv);
      if (row < C) {
        const int i = row;
        const float ri = Rk[i], bi = Bs[i], gi = Gs[i];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int j = c0 + c;
          const float dec = (j <= i) ? __expf(gi - Gs[j]) : 0.0f;
          As[i * LDC + j] = (j < i) ? bi * (ri * gv[c] * Rk[j]) * dec : 0.0f;
        }
      } else if (!TCB) {  // with TCB, phase B forms P itself
        const int i = row - C;
        const float ri = Rq[i], gi = Gs[i];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int j = c0 + c;
          const float dec = (j <= i) ? __expf(gi - Gs[j]) : 0.0f;
          ws[WS::PT + j * WS::LW + i] = (ri * gv[c] * Rk[j]) * dec;
        }
      }
    }
    tc_fence_before_sync();
    __syncthreads();  // A complete; Q consumed; the tile is out of TMEM
    if (warp == 0) {
      tc_fence_after_sync();
      tmem_dealloc(tmem, kTmemCols);
    }
  } else {
    // fp32 inputs: on the tensor cores as warp-level 3xTF32 products of the
    // normalised rows: warp w takes rows 16 (w % 4) .. and the four 8-column
    // blocks from 32 (w / 4)
    {
      const int g = lane >> 2, t = lane & 3;
      const int m0 = (warp & 3) * 16, nb = (warp >> 2) * 32;
      float kk[4][4], qk[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) kk[j][e] = qk[j][e] = 0.0f;
#pragma unroll 2
      for (int k0 = 0; k0 < DK; k0 += 8) {
        uint32_t akh[4], akl[4], aqh[4], aql[4];
        load_a_split_rows(Ks, LDQ, m0, k0, g, t, akh, akl);
        load_a_split_rows(Qs, LDQ, m0, k0, g, t, aqh, aql);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t bh[2], bl[2];
          load_b_split_cols(Ks, LDQ, k0, nb + 8 * j, g, t, bh, bl);
          mma_3xtf32(kk[j], akh, akl, bh, bl);
          mma_3xtf32(qk[j], aqh, aql, bh, bl);
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = m0 + g + 8 * (e >> 1), jj = nb + 8 * j + 2 * t + (e & 1);
          const float dec = (jj <= i) ? __expf(Gs[i] - Gs[jj]) : 0.0f;
          As[i * LDC + jj] = (jj < i) ? Bs[i] * kk[j][e] * dec : 0.0f;
          ws[WS::PT + jj * WS::LW + i] = qk[j][e] * dec;
        }
    }
    write_decayed_qk();
    __syncthreads();  // A complete; Q consumed
  }
  if constexpr (!TCB) {
    // beta_j gamma_j k_j, row-major, into the Q buffer
    for (int e = tid; e < C * DK; e += 256) {
      const int j = e / DK, d = e % DK;
      Qs[j * LDR + d] = Ks[j * LDQ + d] * Eb[j];
    }
    __syncthreads();  // K consumed
    // beta_j v_j, row-major, into the K buffer (loads issued together)
#pragma unroll
    for (int e = tid; e < C * DV / 4; e += 256) {
      const int j = e / (DV / 4), d4 = (e % (DV / 4)) * 4;
      float vv[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      if (j < len)
        load_vec<InT, 4>(
            reinterpret_cast<const InT*>(p.v) + ((size_t)(t0 + j) * p.H + h) * DV + d4, vv);
      *reinterpret_cast<float4*>(Ks + j * LDR + d4) =
          make_float4(vv[0] * Bs[j], vv[1] * Bs[j], vv[2] * Bs[j], vv[3] * Bs[j]);
    }
  }
  // 4. T = (I + A)^-1 into T^T
  invert_unit_lower64<LDC, LDT>(As, Tt, Ys, tid);

  if constexpr (TCB) {
    // 5. T itself, for phase B, in 8 x 8 blocks (tcb_t_index): a thread
    //    writes 4 consecutive floats of a block row, so a warp writes 512
    //    contiguous bytes
    for (int e4 = tid; e4 < C * C / 4; e4 += 256) {
      const int blk = e4 >> 4, r = (e4 >> 1) & 7, m4 = (e4 & 1) * 4;
      const int i = (blk >> 3) * 8 + r, m = (blk & 7) * 8 + m4;
      *reinterpret_cast<float4*>(ws + 4 * e4) =
          make_float4(Tt[m * LDT + i], Tt[(m + 1) * LDT + i], Tt[(m + 2) * LDT + i],
                      Tt[(m + 3) * LDT + i]);
    }
  } else {
    // 5. W = T (diag(beta gamma) K) and U = T (diag(beta) V) on the tensor
    //    cores (3xTF32): T^T is the k-major A operand; warp w takes rows
    //    16 (w % 4) .. and half of the columns
    {
      const int g = lane >> 2, t = lane & 3;
      const int m0 = (warp & 3) * 16;
      {
        constexpr int NB = DK / 16;  // 8-column blocks per warp
        const int nb = (warp >> 2) * NB * 8;
        float w[NB][4];
  #pragma unroll
        for (int j = 0; j < NB; ++j)
  #pragma unroll
          for (int e = 0; e < 4; ++e) w[j][e] = 0.0f;
  #pragma unroll 2
        for (int k0 = 0; k0 < C; k0 += 8) {
          uint32_t ah[4], al[4];
          load_a_split(Tt, LDT, m0, k0, g, t, ah, al);
  #pragma unroll
          for (int j = 0; j < NB; ++j) {
            uint32_t bh[2], bl[2];
            load_b_split(Qs, LDR, k0, nb + 8 * j, g, t, bh, bl);
            mma_3xtf32(w[j], ah, al, bh, bl);
          }
        }
  #pragma unroll
        for (int j = 0; j < NB; ++j)  // W transposed
  #pragma unroll
          for (int e = 0; e < 4; ++e)
            ws[WS::WT + (nb + 8 * j + 2 * t + (e & 1)) * WS::LW + m0 + g + 8 * (e >> 1)] = w[j][e];
      }
      {
        constexpr int NB = DV / 16;
        const int nb = (warp >> 2) * NB * 8;
        float u[NB][4];
  #pragma unroll
        for (int j = 0; j < NB; ++j)
  #pragma unroll
          for (int e = 0; e < 4; ++e) u[j][e] = 0.0f;
  #pragma unroll 2
        for (int k0 = 0; k0 < C; k0 += 8) {
          uint32_t ah[4], al[4];
          load_a_split(Tt, LDT, m0, k0, g, t, ah, al);
  #pragma unroll
          for (int j = 0; j < NB; ++j) {
            uint32_t bh[2], bl[2];
            load_b_split(Ks, LDR, k0, nb + 8 * j, g, t, bh, bl);
            mma_3xtf32(u[j], ah, al, bh, bl);
          }
        }
  #pragma unroll
        for (int j = 0; j < NB; ++j)
  #pragma unroll
          for (int h2 = 0; h2 < 2; ++h2)
            *reinterpret_cast<float2*>(ws + WS::U + (m0 + g + 8 * h2) * WS::LU + nb + 8 * j + 2 * t) =
                make_float2(u[j][2 * h2], u[j][2 * h2 + 1]);
      }
    }
  }
}

// Shared memory of phase B (floats): one chunk's workspace block, copied as
// it is, then the state transposed, S[d][j] (row stride DV + 8: the B
// fragments of a warp hit 32 distinct banks).
template <int DK, int DV>
struct PhaseBSmem {
  static constexpr int LDS = DV + 8;
  static constexpr int WSB = 0;                            // ChunkWs<DK, DV> block
  static constexpr int SS = WSB + ChunkWs<DK, DV>::SIZE;   // [DK][LDS]
  static constexpr int FLOATS = SS + DK * LDS;
  static constexpr size_t BYTES = (size_t)FLOATS * sizeof(float) + 16;  // + the mbarrier
};

// Phase B CTAs are handed out longest sequence first (for up to this many
// sequences; beyond it, in sequence order): with one CTA per SM a long
// sequence started late would otherwise set the end of the launch.
constexpr int kSortSeqMax = 256;

// The sequence of a per-(sequence, head) block: block v takes head v % H of
// the sequence ranked v / H by chunk count (descending, ties in sequence
// order) when there are at most kSortSeqMax sequences, else sequence v / H.
// Every thread of the block calls it (it contains a CTA barrier); `pick` is
// shared memory; the block has at least kSortSeqMax threads.
__device__ __forceinline__ int longest_first_sequence(const int32_t* cu, int N, int H, int total,
                                                      int* pick) {
  int n = (int)(blockIdx.x / (unsigned)H);
  if (N <= kSortSeqMax) {
    const int tid = threadIdx.x;
    if (tid < N) {
      const long long ci = seq_chunks(__ldg(cu + tid), __ldg(cu + tid + 1), total);
      int rank = 0;
      for (int j = 0; j < N; ++j) {
        const long long cj = seq_chunks(__ldg(cu + j), __ldg(cu + j + 1), total);
        rank += (cj > ci || (cj == ci && j < tid)) ? 1 : 0;
      }
      if (rank == n) *pick = tid;
    }
    __syncthreads();
    n = *pick;
  }
  return n;
}

__device__ __forceinline__ int phase_b_sequence(const PrefillParams& p, int* pick) {
  return longest_first_sequence(p.cu_seqlens, p.N, p.H, p.total, pick);
}

// Phase B: the state through the chunks.  Grid N * H; 256 threads (8
// warps); every product on the tensor cores in 3xTF32:
//   Delta = U - W S  and  QG S       (C x DV)  warp: one 16-row block, DV/16 columns
//   O     = scale (QG S + P Delta)
//   S    <- gamma_C S + KD^T Delta   (DK x DV) warp: DK/8 ... see NT3
template <int DK, int DV, typename OutT>
__global__ void __launch_bounds__(256, 1) prefill_state_kernel(const PrefillParams p) {
  constexpr int C = kChunk, NT = 256;
  using SM = PhaseBSmem<DK, DV>;
  using WS = ChunkWs<DK, DV>;
  constexpr int LDS = SM::LDS, LW = WS::LW, LU = WS::LU, LKD = WS::LKD;
  // products 1-2: 4 row blocks of 16 x (DV/8 column blocks of 8); 2 warps per row block
  constexpr int NT1 = DV / 8 / 2;
  // product 3: DK/16 row blocks; 8 warps share them; column blocks split the rest
  constexpr int MB3 = DK / 16, WPM3 = 8 / MB3, NT3 = DV / 8 / WPM3;
  static_assert(C / 16 * 2 == 8 && MB3 * WPM3 == 8 && NT3 * WPM3 * 8 == DV, "warp tiling");
  constexpr unsigned WS_BYTES = WS::SIZE * sizeof(float);
  extern __shared__ __align__(128) float sm[];
  float* wsb = sm + SM::WSB;
  const float* Wt = wsb + WS::WT;
  float* Us = wsb + WS::U;  // U, then Delta in place
  const float* QGt = wsb + WS::QGT;
  const float* KD = wsb + WS::KD;
  const float* Pt = wsb + WS::PT;
  float* Ss = sm + SM::SS;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + SM::FLOATS);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  // block v takes head v % H of the sequence ranked v / H by chunk count
  // (descending, ties in sequence order)
  const int h = (int)(blockIdx.x % (unsigned)p.H);
  __shared__ int pick;
  const int n = phase_b_sequence(p, &pick);
  const int t0 = __ldg(p.cu_seqlens + n), t1 = __ldg(p.cu_seqlens + n + 1);
  OutT* out = reinterpret_cast<OutT*>(p.out);
  if (t0 < 0 || t1 < t0 || t1 > p.total) {
    if (p.dev_status != nullptr && threadIdx.x == 0) atomicOr(p.dev_status, GDN_STATUS_SEQ_RANGE);
    return;
  }
  const int s = __ldg(p.slot_idx + n);
  if (s < 0 || s >= p.n_slots) {
    if (s != -1 && p.dev_status != nullptr && tid == 0) atomicOr(p.dev_status, GDN_STATUS_SLOT_RANGE);
    for (int e = tid; e < (t1 - t0) * DV; e += NT)
      store_scalar(out + ((size_t)(t0 + e / DV) * p.H + h) * DV + e % DV, 0.0f);
    return;
  }

  const long long x0 = first_chunk(p.cu_seqlens, n, p.total);
  const int nc = (t1 - t0 + C - 1) / C;
  const float* ws0 = p.ws + ((size_t)x0 * p.H + h) * WS::SIZE;
  const size_t chunk_stride = (size_t)p.H * WS::SIZE;
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    if (nc > 0) {
      mbar_arrive_expect_tx(bar, WS_BYTES);
      bulk_copy_g2s(wsb, ws0, WS_BYTES, bar);
    }
    if (nc > 1) prefetch_l2(ws0 + chunk_stride, WS_BYTES);
  }

  // the state: pool rows j (dk contiguous) -> Ss[d][j]
  float* pool = p.state + ((size_t)s * p.H + h) * DV * DK;
  for (int e = tid; e < DV * DK; e += NT) {
    const int j = e / DK, d = e % DK;
    Ss[d * LDS + j] = p.initial_state ? pool[e] : 0.0f;
  }

  const int m1 = (warp & 3) * 16, n1 = (warp >> 2) * NT1 * 8;      // products 1-2
  const int m3 = (warp % MB3) * 16, n3 = (warp / MB3) * NT3 * 8;   // product 3
  for (int ch = 0; ch < nc; ++ch) {
    const int len = min(C, t1 - t0 - ch * C);
    // this chunk's block (thread 0 waits, with a bound; the barrier passes it on)
    __shared__ int landed;
    if (tid == 0) landed = mbar_wait_bounded(bar, ch & 1, kWaitLimitNs) ? 1 : 0;
    __syncthreads();
    if (!landed) {
      // report, give the copy one more bounded wait so the shared memory is
      // not released under it, and leave the state as it was
      if (tid == 0) {
        if (p.dev_status != nullptr) atomicOr(p.dev_status, GDN_STATUS_TIMEOUT);
        mbar_wait_bounded(bar, ch & 1, kWaitLimitNs);
      }
      return;
    }
    mbar_try_wait(bar, ch & 1);  // completed: every thread acquires the copied bytes
    const float gamma_c = wsb[WS::GL];

    // 1. W S and QG S on this warp's 16 rows and NT1 column blocks
    float ws_[NT1][4], qs_[NT1][4];
#pragma unroll
    for (int j = 0; j < NT1; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) ws_[j][e] = qs_[j][e] = 0.0f;
#pragma unroll 2
    for (int k0 = 0; k0 < DK; k0 += 8) {
      uint32_t awh[4], awl[4], aqh[4], aql[4];
      load_a_split(Wt, LW, m1, k0, g, t, awh, awl);
      load_a_split(QGt, LW, m1, k0, g, t, aqh, aql);
#pragma unroll
      for (int j = 0; j < NT1; ++j) {
        uint32_t bh[2], bl[2];
        load_b_split(Ss, LDS, k0, n1 + j * 8, g, t, bh, bl);
        mma_3xtf32(ws_[j], awh, awl, bh, bl);
        mma_3xtf32(qs_[j], aqh, aql, bh, bl);
      }
    }
    // Delta = U - W S, in place of U
#pragma unroll
    for (int j = 0; j < NT1; ++j) {
      float* u0 = Us + (m1 + g) * LU + n1 + j * 8 + 2 * t;
      float* u1 = u0 + 8 * LU;
      u0[0] -= ws_[j][0];
      u0[1] -= ws_[j][1];
      u1[0] -= ws_[j][2];
      u1[1] -= ws_[j][3];
    }
    __syncthreads();  // Delta complete; nothing reads S until the update below

    // 2. O = scale (QG S + P Delta) for the chunk's tokens
#pragma unroll 2
    for (int k0 = 0; k0 < C; k0 += 8) {
      uint32_t ah[4], al[4];
      load_a_split(Pt, LW, m1, k0, g, t, ah, al);
#pragma unroll
      for (int j = 0; j < NT1; ++j) {
        uint32_t bh[2], bl[2];
        load_b_split(Us, LU, k0, n1 + j * 8, g, t, bh, bl);
        mma_3xtf32(qs_[j], ah, al, bh, bl);
      }
    }
#pragma unroll
    for (int j = 0; j < NT1; ++j) {
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
        const int i = m1 + g + 8 * hlf;
        if (i < len) {
          OutT* o = out + ((size_t)(t0 + ch * C + i) * p.H + h) * DV + n1 + j * 8 + 2 * t;
          store_scalar(o, p.scale * qs_[j][2 * hlf]);
          store_scalar(o + 1, p.scale * qs_[j][2 * hlf + 1]);
        }
      }
    }

    // 3. S <- gamma_C S + KD^T Delta (each thread updates only its own elements)
    float sn[NT3][4];
#pragma unroll
    for (int j = 0; j < NT3; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) sn[j][e] = 0.0f;
#pragma unroll 2
    for (int k0 = 0; k0 < C; k0 += 8) {
      uint32_t ah[4], al[4];
      load_a_split(KD, LKD, m3, k0, g, t, ah, al);
#pragma unroll
      for (int j = 0; j < NT3; ++j) {
        uint32_t bh[2], bl[2];
        load_b_split(Us, LU, k0, n3 + j * 8, g, t, bh, bl);
        mma_3xtf32(sn[j], ah, al, bh, bl);
      }
    }
#pragma unroll
    for (int j = 0; j < NT3; ++j) {
      float* s0 = Ss + (m3 + g) * LDS + n3 + j * 8 + 2 * t;
      float* s1 = s0 + 8 * LDS;
      s0[0] = fmaf(gamma_c, s0[0], sn[j][0]);
      s0[1] = fmaf(gamma_c, s0[1], sn[j][1]);
      s1[0] = fmaf(gamma_c, s1[0], sn[j][2]);
      s1[1] = fmaf(gamma_c, s1[1], sn[j][3]);
    }
    fence_proxy_async_smem();  // this thread's reads and writes of the block come first
    __syncthreads();           // every access to the block is done: the next copy may land
    if (tid == 0 && ch + 1 < nc) {
      const float* nxt = ws0 + (size_t)(ch + 1) * chunk_stride;
      mbar_arrive_expect_tx(bar, WS_BYTES);
      bulk_copy_g2s(wsb, nxt, WS_BYTES, bar);
      if (ch + 2 < nc) prefetch_l2(nxt + chunk_stride, WS_BYTES);
    }
  }
  __syncthreads();
  for (int e = tid; e < DV * DK; e += NT) {
    const int j = e / DK, d = e % DK;
    pool[e] = Ss[d * LDS + j];
  }
}

}  // namespace gdn
