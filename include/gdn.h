/*
 * gdn.h - C ABI of the B200 (sm_100a) gated delta rule decode library.
 *
 * What is computed (the batched Gated DeltaNet recurrent update at decode
 * time; "GDN tuning limits on Kunlun XPU", section 二 背景, describes it as a
 * per-token rank-1 update of a 128x128-per-head state together with a decay
 * term, inside the chain input projection -> short conv (kernel size 4) ->
 * gating -> recurrence -> output projection).  For every sequence b, v-head h
 * and token t, with S the dk x dv state of (slot_idx[b], h):
 *
 *     alpha = exp(g[b,t,h])              (g <= 0 gives alpha in (0, 1])
 *     S     = alpha * S                               decay
 *     delta = beta[b,t,h] * (v[b,t,h] - S^T k)        delta-rule prediction
 *     S     = S + k delta^T                           rank-1 update
 *     o     = scale * S^T q                           read-out
 *
 * where q and k are the (L2-normalised, by default) vectors of q/k head
 * h / (H/Hk).  Tokens t = 0..T-1 are applied in order; the state is read from
 * and written to HBM once per call.
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are caller-owned DEVICE memory, dense row-major in
 *    the layouts given below.  The library allocates nothing on these paths
 *    and keeps no per-call state; pools are updated in place.
 *  - State storage layout: state[slot][h][j][i] = S_ij, i in [0,dk) fastest.
 *    A dv column of S is therefore one contiguous dk-float row.
 *  - slot_idx[b] selects the state slot of sequence b.  -1 marks a padding
 *    row: its out rows are written as zeros and no state (or conv state) is
 *    read or written.  Non-negative entries must be unique; duplicates are a
 *    caller error (the result is then unspecified) and are detected only when
 *    slot checking is on (see gdn_step_args.check_slots / GDN_DEBUG=1).
 *  - A slot outside [-1, n_slots) is never dereferenced: its rows are treated
 *    as padding and GDN_STATUS_SLOT_RANGE is OR-ed into *dev_status (when a
 *    status word is given).  No kernel traps.
 *  - Calls are asynchronous: they enqueue kernels on `stream` (a
 *    cudaStream_t; NULL = legacy default stream) and return.  Host-side
 *    argument errors return synchronously before anything is enqueued.
 *  - Return value: GDN_OK (0) or a negative gdn_status.  The message of the
 *    last error on the calling thread is available from
 *    gdn_last_error_string().
 *  - Supported shapes: dk in {64, 128}; dv in {64, 128}; T in [1, 8];
 *    H % Hk == 0.  B == 0 is a no-op.
 *  - Alignment: state, q, k, v and out must be 16-byte aligned.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { GDN_F32 = 0, GDN_BF16 = 1, GDN_F16 = 2 } gdn_dtype;

typedef enum {
  GDN_OK = 0,
  GDN_ERR_ARG = -1,          /* null pointer, bad size, misalignment, bad enum */
  GDN_ERR_UNSUPPORTED = -2,  /* valid but not built: dk/dv/T/group outside the set above */
  GDN_ERR_CUDA = -3,         /* a CUDA runtime call failed; see gdn_last_error_string() */
  GDN_ERR_SLOT_RANGE = -4,   /* a slot outside [-1, n_slots) */
  GDN_ERR_SLOT_DUP = -5,     /* two batch rows name the same non-negative slot */
  GDN_ERR_ACCEPT_RANGE = -6, /* an n_accept entry outside [0, T] */
  GDN_ERR_SEQ_RANGE = -7,    /* a prefill sequence's tokens outside [0, total_tokens] */
  GDN_ERR_TIMEOUT = -8       /* a kernel gave up waiting for its own copy */
} gdn_status;

/* Bits OR-ed into the optional device status word by the kernels.
 *
 * The only waits in the library are kernels waiting for their own work: the
 * multi-token block form (calls of 2..4 tokens on an fp32 pool), the staged
 * single-token kernel (16-bit pools, dk = 128) and the low-rank kernel wait
 * for their bulk copy into shared memory; the tensor-core block form (calls
 * of 2..4 tokens on a 16-bit pool, dk = dv = 128) and the chunked prefill
 * wait for their copies and their tensor-core products.  Each wait gives up
 * after one second and sets GDN_STATUS_TIMEOUT: the decode kernels then skip
 * that tile or head (its state is left as it was, its outputs are not
 * written); the tensor-core block form, whose CTAs each walk several heads,
 * also skips the heads that CTA had not reached; the prefill leaves that
 * chunk's work undone.
 * After GDN_STATUS_TIMEOUT treat every later result on the device as
 * untrusted until the stream has been drained: an operation that was
 * given up on may still complete afterwards.
 *
 * The other device-side conditions are bad indices: a slot outside
 * [-1, n_slots) (GDN_STATUS_SLOT_RANGE), an n_accept entry outside [0, T]
 * (GDN_STATUS_ACCEPT_RANGE), or a prefill sequence whose token range is not
 * inside [0, total_tokens] (GDN_STATUS_SEQ_RANGE: the sequence is skipped,
 * its outputs and state untouched). */
#define GDN_STATUS_SLOT_RANGE 0x1
#define GDN_STATUS_ACCEPT_RANGE 0x2
#define GDN_STATUS_SEQ_RANGE 0x4
#define GDN_STATUS_TIMEOUT 0x8

/*
 * gdn_decode_step - the batched decode step with its default options.
 *
 *   q, k     bf16 [B][T][H][dk]       (Hk = H: one q/k head per v-head)
 *   v        bf16 [B][T][H][dv]
 *   g        fp32 [B][T][H]           log decay; alpha = exp(g)
 *   beta     fp32 [B][T][H]           delta-rule step size (already sigmoid-ed)
 *   state    fp32 pool [n_slots][H][dv][dk], read and written in place
 *   slot_idx int32 [B]
 *   out      fp32 [B][T][H][dv]
 *   stream   cudaStream_t (may be NULL)
 *
 * Fixed options: q and k are L2-normalised inside the kernel with
 * x / sqrt(sum x^2 + 1e-6); scale = 1/sqrt(dk); the pool size is not known,
 * so only slot >= -1 is checked (the caller guarantees slot < n_slots).
 */
GDN_API int gdn_decode_step(const void* q, const void* k, const void* v,
                    const float* g, const float* beta, float* state,
                    const int32_t* slot_idx, float* out, int B, int H, int dk,
                    int dv, int T, void* stream);

/*
 * gdn_decode_step_ex - the same step with every option explicit.
 *
 *   q, k      in_dtype [B][T][Hk][dk]; v in_dtype [B][T][H][dv]
 *             (in_dtype: GDN_F32 or GDN_BF16)
 *   g, beta   fp32 [B][T][H]
 *   state     state_dtype [n_slots][H][dv][dk]
 *   out       out_dtype [B][T][H][dv] (GDN_F32 or GDN_BF16)
 *   state_dtype  GDN_F32 (default), or GDN_BF16 / GDN_F16 for a 16-bit
 *             state pool: rows are widened to fp32 on load, every token is
 *             computed in fp32, and the state is rounded to nearest-even
 *             into the pool once, at the end of the call (half the HBM
 *             bytes of an fp32 pool).  16-bit pools need dk / 8 lanes, i.e.
 *             any supported dk.
 *   n_slots   pool size; slots outside [-1, n_slots) are reported, not used.
 *             n_slots <= 0 means "unknown" (only slot >= -1 is checked).
 *             Calls of 2..4 tokens on a 16-bit pool with dk = dv = 128 run
 *             on the tensor cores with the pool described to the TMA unit,
 *             which needs its extent: with n_slots <= 0 (or a pool of 2^31
 *             rows or more) they take the token loop instead (same results
 *             to the pool's rounding, slower).
 *   scale     read-out scale; <= 0 selects 1/sqrt(dk).
 *   qk_l2norm 1: normalise q and k in the kernel (eps below); 0: use as given.
 *   l2_eps    epsilon inside the L2 norm's square root (1e-6 if < 0).
 *   dev_status  nullable device int; kernels atomicOr GDN_STATUS_* bits into
 *             it and never clear it.  Read it with gdn_get_error().
 *   check_slots 1: before launching, copy slot_idx (and token_slots) to
 *             the host (this synchronises `stream`) and return
 *             GDN_ERR_SLOT_RANGE / GDN_ERR_SLOT_DUP without launching if the
 *             slots are out of range, repeated, or a token slot is also a
 *             source slot.  Also enabled for every call when the environment
 *             has GDN_DEBUG=1.
 *
 * Bits of a T-token call against T one-token calls on an fp32 pool (each
 * kernel fixes its rounding order; the bits do not depend on the batch, the
 * slots or the other rows):
 *   - T = 1 and T = 5..8: the tokens are applied one at a time with the
 *     arithmetic of a one-token call, so the outputs and the stored state
 *     are bit-identical to T consecutive one-token calls.
 *   - T = 2..4: the call takes all its tokens against the starting state at
 *     once (the unrolled recurrence).  The first token's output carries the
 *     bits of a one-token call; the later tokens' outputs and the stored
 *     state agree with T one-token calls to fp32 rounding (a few ulps), not
 *     bit for bit.  A call with n_accept = n (or a token_slots snapshot
 *     after token n) stores exactly the bits of an n-token call.
 *   Callers that replay accepted tokens one by one and need the bits of the
 *   verify pass should therefore commit through n_accept / token_slots.
 * On a bf16 / fp16 pool the state is rounded to the pool's type once per
 * call, so T one-token calls (which round T times) differ from one T-token
 * call by that rounding; both stay within one storage ulp of the exact
 * recurrence per call.  With dk = dv = 128 and T = 2..4 a call runs the block
 * form on the tensor cores, except with token_slots (the token loop): the
 * outputs of the two agree to fp32 rounding, not bit for bit; n_accept does
 * not change the outputs' bits.
 *
 * Speculative decoding (multi-token verify; at most one of the two):
 *   n_accept  nullable int32 [B]: outputs are produced for all T tokens, but
 *             the state stored back in slot_idx[b] is the state after the
 *             first n_accept[b] tokens; n_accept[b] == 0 leaves the slot
 *             unwritten (a read-only verify pass).  An entry outside [0, T]
 *             writes nothing and sets GDN_STATUS_ACCEPT_RANGE.
 *   token_slots  nullable int32 [B][T]: per-token snapshots.  The state
 *             after token t is stored in pool slot token_slots[b][t] (-1:
 *             not stored) and slot_idx[b] is not written, so accepting a
 *             prefix of n tokens is a matter of making token_slots[b][n-1]
 *             the sequence's slot.  Token slots must be distinct and must
 *             not be any row's source slot (a caller error otherwise); a
 *             slot outside [-1, n_slots) is skipped and reported with
 *             GDN_STATUS_SLOT_RANGE.
 */
typedef struct {
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const float* beta;
  void* state;
  const int32_t* slot_idx;
  void* out;
  int B, Hk, H, dk, dv, T, n_slots;
  gdn_dtype in_dtype;     /* dtype of q, k, v */
  gdn_dtype out_dtype;    /* dtype of out */
  gdn_dtype state_dtype;  /* dtype of the state pool */
  float scale;
  int qk_l2norm;
  float l2_eps;
  int* dev_status;
  int check_slots;
  const int32_t* n_accept;
  const int32_t* token_slots;
  void* stream;
} gdn_step_args;

GDN_API int gdn_decode_step_ex(const gdn_step_args* a);

/*
 * gdn_fused_decode_step - one decode token (T = 1) with the layer's front
 * and epilogue fused around the recurrence ("GDN tuning limits on Kunlun
 * XPU", section 二 背景: short conv of kernel size 4 and gating before the
 * recurrence; the gated output o * silu(z) after it):
 *
 *   1. causal depthwise conv, kernel 4, no bias, then SiLU, over every
 *      channel c of the mixed projection row x = mixed_x[b] (C channels,
 *      ordered [q: Hk*dk | k: Hk*dk | v: H*dv]):
 *          y_c = silu(w[c][0]*cs[c][0] + w[c][1]*cs[c][1] + w[c][2]*cs[c][2]
 *                     + w[c][3]*x_c)
 *      where cs = conv_state[slot] holds the three previous inputs, oldest
 *      first; afterwards cs[c] = {cs[c][1], cs[c][2], x_c}.
 *   2. q, k = L2-normalised (eps 1e-6) q/k channels of k-head h / (H/Hk);
 *      v = the v channels of v-head h.
 *   3. g = -exp(A_log[h]) * softplus(a[b][h] + dt_bias[h]);
 *      beta = sigmoid(b[b][h]).
 *   4. the recurrence above with scale = 1/sqrt(dk).
 *   5. out[b][h][j] = o_j / sqrt(mean_j(o^2) + norm_eps) * norm_w[j]
 *                     * silu(z[b][h*dv + j]).
 *
 *   mixed_x    bf16 [B][C];  conv_state bf16 [n_slots][C][3] (in place)
 *   conv_w     conv_w_dtype [C][4]
 *   a, b       bf16 [B][H];  A_log, dt_bias fp32 [H]
 *   z          bf16 [B][H*dv];  norm_w fp32 [dv]
 *   state      fp32 [n_slots][H][dv][dk] (in place);  slot_idx int32 [B]
 *   out        out_dtype [B][H][dv]
 *   n_slots    pool size (required, > 0)
 *   dev_status nullable, as in gdn_decode_step_ex.
 * Requirements beyond the common ones: H / Hk <= 8; mixed_x, z and out
 * 16-byte aligned; conv_w 16-byte (fp32) or 8-byte (bf16) aligned.
 */
GDN_API int gdn_fused_decode_step(const void* mixed_x, void* conv_state,
                          const void* conv_w, gdn_dtype conv_w_dtype,
                          const void* a, const void* b, const float* A_log,
                          const float* dt_bias, const void* z,
                          const float* norm_w, float norm_eps, float* state,
                          const int32_t* slot_idx, void* out, int B, int Hk,
                          int H, int dk, int dv, int n_slots,
                          gdn_dtype out_dtype, int* dev_status, void* stream);

/*
 * gdn_chunk_prefill - the same recurrence over whole prompts (prefill).
 *
 * N sequences are packed along the token axis: sequence n owns tokens
 * [cu_seqlens[n], cu_seqlens[n+1]).  Every (sequence, head) starts from pool
 * slot slot_idx[n] (or from a zero state when initial_state == 0), applies
 * its tokens in order exactly as gdn_decode_step does, writes every token's
 * output, and stores its final state back in that slot.  slot_idx[n] == -1
 * skips the sequence (its outputs are zero, no state is touched).
 *
 * The tokens are processed in chunks of 64 with the chunkwise form of the
 * recurrence (per chunk, with gamma_i the decay accumulated from the chunk
 * start: Delta = (I + A)^-1 diag(beta)(V - diag(gamma) K S0) with
 * A_ij = beta_i (k_i.k_j) gamma_i/gamma_j for j < i; outputs
 * scale (diag(gamma) Q S0 + P Delta); end state gamma_C S0 +
 * (K gamma_C/gamma)^T Delta), to fp32 accuracy.  Two kernels: the first
 * forms every chunk's (I + A)^-1 (and, on the general path, the other chunk
 * matrices) in parallel; the second carries the state through each
 * sequence's chunks.  With bf16 inputs and dk = dv = 128 every product runs
 * on the 5th-generation tensor cores (tcgen05), fp32 operands split into
 * bf16 parts; other inputs and head sizes use warp-level tensor-core
 * products in 3xTF32.
 *
 *   q, k       in_dtype [total_tokens][Hk][dk];  v in_dtype [total_tokens][H][dv]
 *   g, beta    fp32 [total_tokens][H]
 *   state      fp32 pool [n_slots][H][dv][dk] (read and written in place)
 *   slot_idx   int32 [N];  cu_seqlens int32 [N+1], device memory, non-decreasing,
 *              cu_seqlens[N] <= total_tokens
 *   out        out_dtype [total_tokens][H][dv] (rows of padding sequences
 *              are zero; rows past cu_seqlens[N] are not written)
 *   workspace  device scratch of at least gdn_prefill_workspace_size_ex(...)
 *              bytes for the call's in_dtype (gdn_prefill_workspace_size
 *              covers either dtype), 16-byte aligned, owned by the caller; its contents
 *              need no initialisation and are meaningless afterwards.
 *              Two prefill calls that may run concurrently need two
 *              workspaces.
 * Supported: dk, dv in {64, 128}; H % Hk == 0.  Asynchronous on `stream`
 * (two kernel launches).
 */
typedef struct {
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const float* beta;
  float* state;
  const int32_t* slot_idx;
  const int32_t* cu_seqlens;
  void* out;
  int N, total_tokens, Hk, H, dk, dv, n_slots;
  gdn_dtype in_dtype;
  gdn_dtype out_dtype;
  float scale;         /* <= 0 -> 1/sqrt(dk) */
  int qk_l2norm;       /* 1 = normalise q, k (eps below) */
  float l2_eps;        /* < 0 -> 1e-6 */
  int initial_state;   /* 1: start from the slot's state; 0: from zeros */
  void* workspace;
  size_t workspace_bytes;
  int* dev_status;     /* nullable, as in gdn_decode_step_ex */
  void* stream;
} gdn_prefill_args;

/* Bytes of workspace gdn_chunk_prefill needs for N sequences of
 * total_tokens tokens in all with inputs of type in_dtype (an upper bound
 * that does not depend on how the tokens are split).  bf16 inputs with
 * dk = dv = 128 need 16 KiB per chunk slot and head (the chunk's
 * (I + A)^-1 only); other inputs and head sizes need the chunk matrices of
 * the general path (about 158 KiB at dk = dv = 128).  Returns 0 for
 * unsupported sizes or dtypes. */
GDN_API size_t gdn_prefill_workspace_size_ex(int N, int total_tokens, int H, int dk, int dv,
                                             gdn_dtype in_dtype);

/* The same bound for any input dtype (the larger of the two). */
GDN_API size_t gdn_prefill_workspace_size(int N, int total_tokens, int H, int dk, int dv);

GDN_API int gdn_chunk_prefill(const gdn_prefill_args* a);

/*
 * gdn_chunk_prefill_noalloc - gdn_chunk_prefill without a caller workspace.
 * (An interface of this library; the pages have no counterpart.)
 *
 * For callers that cannot obtain device memory at the time of the call:
 * for example a host program that hands this library only pre-planned
 * tensors and owns every allocation itself, an engine whose memory budget
 * is fixed when it starts, or a code path that must not enter the CUDA
 * allocator.  Instead of the `workspace` fields (which are ignored), the
 * call uses a scratch array of 64 MiB that is part of the library's device
 * image: every GPU that loads the library holds those 64 MiB until the
 * process exits.  Nothing is allocated or freed by the call.
 *
 *  - Limit: the call needs gdn_prefill_workspace_size_ex(N, total_tokens, H,
 *    dk, dv, in_dtype) <= 64 MiB, with total_tokens / 64 + N + 1 chunk
 *    slots per head.  With bf16 inputs at dk = dv = 128 that is 4096 chunk
 *    slots times heads: for example one prompt of up to 5375 tokens with 48
 *    heads; with fp32 inputs at dk = dv = 128, 414 (one prompt of up to 447
 *    tokens with 48 heads).  A larger request returns GDN_ERR_UNSUPPORTED
 *    with the sizes in the message.
 *  - The first call on a device looks up the scratch array's device address
 *    (cudaGetSymbolAddress, with that device current) and keeps it; make
 *    that first call before capturing any stream on that device.  The kept
 *    address belongs to the device's primary context (the one the CUDA
 *    runtime uses): it is not valid in another context made current
 *    through the driver API, nor after cudaDeviceReset on that device.
 *  - Every call on a device shares the one array, and it keeps whatever the
 *    last call wrote.  This is harmless here because a prefill writes every
 *    scratch value before reading it.  But two calls whose work may overlap
 *    on the GPU (different streams without ordering between them) race on
 *    the scratch and give wrong results: order them.
 * Everything else (arguments, layouts, results, errors) is as for
 * gdn_chunk_prefill.
 */
GDN_API int gdn_chunk_prefill_noalloc(const gdn_prefill_args* a);

/*
 * gdn_lowrank_decode_step - decode with a low-rank sliding-window state.
 * ("GDN tuning limits on Kunlun XPU", section 三.3: the low-rank state is a
 * cache of the most recent r rank-1 updates, not a matrix factorisation.)
 *
 * The state of (slot, head) is a window of its R most recent updates
 * (k_j, u_j) with the decay c_j accumulated since each was made; it stands
 * for S = sum_j c_j k_j u_j^T.  Per token, with q, k normalised as in
 * gdn_decode_step: c_j <- alpha c_j; p = sum_j c_j (k_j.k) u_j;
 * delta = beta (v - p); (k, delta) is pushed with c = 1, replacing the
 * oldest entry when the window is full; o = scale sum_j c_j (k_j.q) u_j over
 * the new window.  While the window has never been full this is exactly the
 * full-rank step started from a zero state.
 *
 *   q, k        in_dtype [B][T][Hk][dk];  v in_dtype [B][T][H][dv]
 *   g, beta     fp32 [B][T][H]
 *   win_k       fp32 [n_slots][H][R][dk]   cached k_j (ring order)
 *   win_u       fp32 [n_slots][H][R][dv]   cached u_j (= delta_j)
 *   win_c       fp32 [n_slots][H][R]       decay weights c_j
 *   win_count   int32 [n_slots][H]         updates made so far; update n
 *               lives in ring position n % R.  A fresh sequence starts with
 *               win_count = 0 (the window contents are then never read).
 *   out         out_dtype [B][T][H][dv]
 * Supported: R in {8, 16, 32, 64}; dk, dv in {64, 128}; T in [1, 8].
 * Padding / out-of-range slots behave as in gdn_decode_step_ex.
 */
typedef struct {
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const float* beta;
  float* win_k;
  float* win_u;
  float* win_c;
  int32_t* win_count;
  const int32_t* slot_idx;
  void* out;
  int B, Hk, H, dk, dv, T, R, n_slots;
  gdn_dtype in_dtype;
  gdn_dtype out_dtype;
  float scale;     /* <= 0 -> 1/sqrt(dk) */
  int qk_l2norm;
  float l2_eps;    /* < 0 -> 1e-6 */
  int* dev_status;
  void* stream;
} gdn_lowrank_args;

GDN_API int gdn_lowrank_decode_step(const gdn_lowrank_args* a);

/*
 * gdn_lowrank_prefill - the low-rank window over whole prompts.
 * ("GDN tuning limits on Kunlun XPU", section 三.3, runs the low-rank chain
 * over a prompt in chunks.)
 *
 * N sequences are packed along the token axis as in gdn_chunk_prefill:
 * sequence n owns tokens [cu_seqlens[n], cu_seqlens[n+1]).  The window of
 * (slot_idx[n], h) takes the sequence's tokens in order exactly as
 * gdn_lowrank_decode_step takes the tokens of a call, from the window stored
 * in the slot (initial_window = 1) or from an empty one (0: the slot's
 * count is taken as 0); every token's output is written and the window left
 * behind (the R most recent updates, their decay weights, the count) is
 * stored in the slot.  slot_idx[n] == -1 skips the sequence (zero outputs,
 * no window touched).
 *
 * The tokens run in chunks of 64: within a chunk the updates form a banded
 * lower-triangular system (each token's prediction sees the R updates
 * before it), solved with the chunk's unit lower-triangular inverse, in
 * fp32 on the CUDA cores; one CTA per (sequence, head) carries the window
 * from chunk to chunk.
 *
 *   q, k   in_dtype [total_tokens][Hk][dk];  v in_dtype [total_tokens][H][dv]
 *   g, beta  fp32 [total_tokens][H]
 *   win_k, win_u, win_c, win_count  as in gdn_lowrank_args (in place)
 *   slot_idx int32 [N]; cu_seqlens int32 [N+1] (device, non-decreasing,
 *            cu_seqlens[N] <= total_tokens)
 *   out    out_dtype [total_tokens][H][dv] (rows past cu_seqlens[N] are not
 *          written)
 * Supported: R in {8, 16, 32, 64}; dk, dv in {64, 128}; H % Hk == 0.  Needs
 * no workspace.  Errors and status bits as in gdn_chunk_prefill.
 */
typedef struct {
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const float* beta;
  float* win_k;
  float* win_u;
  float* win_c;
  int32_t* win_count;
  const int32_t* slot_idx;
  const int32_t* cu_seqlens;
  void* out;
  int N, total_tokens, Hk, H, dk, dv, R, n_slots;
  gdn_dtype in_dtype;
  gdn_dtype out_dtype;
  float scale;         /* <= 0 -> 1/sqrt(dk) */
  int qk_l2norm;
  float l2_eps;        /* < 0 -> 1e-6 */
  int initial_window;  /* 1: continue the slot's window; 0: start empty */
  int* dev_status;
  void* stream;
} gdn_lowrank_prefill_args;

GDN_API int gdn_lowrank_prefill(const gdn_lowrank_prefill_args* a);

/*
 * gdn_get_error - read a device status word written by the kernels.
 * Copies *dev_status to *host_status with a blocking cudaMemcpy (so it waits
 * for work already enqueued on the legacy stream; synchronise other streams
 * first).  Returns GDN_OK if no bit is set, GDN_ERR_SLOT_RANGE if
 * GDN_STATUS_SLOT_RANGE is set, else GDN_ERR_ACCEPT_RANGE, GDN_ERR_SEQ_RANGE
 * or GDN_ERR_TIMEOUT for those bits; GDN_ERR_ARG for null pointers and
 * GDN_ERR_CUDA if the copy fails.  Does not clear the word.
 */
GDN_API int gdn_get_error(const int* dev_status, int* host_status);

/* Message of the last error returned on the calling thread ("" if none).
 * The pointer stays valid until the thread's next failing call. */
GDN_API const char* gdn_last_error_string(void);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
GDN_API int gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
