/*
 * libcattn -- fused causal multi-head self-attention for NVIDIA B200 (sm_100a).
 *
 * What is computed.  For every batch b and head h independently
 * ("nanoGPT: a real GPT in two 300-line files", section 2 "How the code
 * works", CausalSelfAttention: one head per slice, attention on its own
 * slice, heads glued back together):
 *
 *     S   = scale * Q K^T                  (T x T, never stored)
 *     S_ij = -inf for j > i                ("fill the future with -inf";
 *                                           "Causal" in "Words to know":
 *                                           a position sees itself and
 *                                           earlier positions only)
 *     P   = softmax(S) row-wise
 *     O   = P V
 *     LSE_i = log(sum_{j<=i} exp(S_ij))    (natural log)
 *
 * "The 300-Line LLM Engine: Inside nanoGPT" ("Flat Architecture and Flash
 * Attention") names not materialising that T x T matrix as the source of
 * the model's speed; no call here ever writes an S- or P-sized buffer.
 *
 * Conventions common to every call:
 *  - Q, K, V, O, dO, dQ, dK, dV are caller-owned DEVICE pointers to bf16
 *    (__nv_bfloat16) tensors of shape (B, H, T, D), contiguous, row-major
 *    (D fastest), 16-byte aligned.  LSE and Delta are caller-owned device
 *    fp32 tensors of shape (B, H, T), contiguous, 4-byte aligned.
 *  - T_q = T_k = T.  Causality is always on; there is no dropout and no
 *    mask argument.  D must be 16, 32, 64 or 128; B, H, T >= 0 with
 *    B*H <= 2^31-1 and T <= 2^20.  A shape with B*H*T == 0 is empty: the
 *    call checks its other scalar arguments, launches nothing and returns
 *    CATTN_OK (pointers may then be NULL).
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  All
 *    work is asynchronous on that stream; a return of CATTN_OK means the
 *    arguments were valid and every launch was accepted, nothing more.
 *  - On any error return nothing has been launched and no output has
 *    been touched.
 *  - The library allocates no device memory for these calls and keeps no
 *    per-call state.  Kernels whose internal waits exceed their poll limit
 *    (a hang guard) record CATTN_ERR_TIMEOUT and exit.  A backward call
 *    records it in status words at the start of its own workspace (read
 *    them with cattn_last_device_status(workspace, stream)), so calls on
 *    different workspaces keep separate records; every kernel also records
 *    it in one library-global device word (cattn_get_device_status()),
 *    which is the only record a forward call has, its signature having no
 *    workspace.
 *  - Per-device set-up the library caches (kernel attributes, the address
 *    of attn_bwd_noalloc's array) belongs to the device's primary CUDA
 *    context.  After cudaDeviceReset() or any other destruction of that
 *    context, unload the library (or restart the process) before calling
 *    it again on that device.
 */
#ifndef CATTN_H
#define CATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CATTN_API __attribute__((visibility("default")))
#else
#define CATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CATTN_OK = 0,
  CATTN_ERR_INVALID_ARG = 1, /* null pointer, bad size, misalignment, small workspace */
  CATTN_ERR_UNSUPPORTED = 2, /* head size D not instantiated; device not sm_100 */
  CATTN_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
  CATTN_ERR_TIMEOUT = 4,     /* a kernel's bounded wait ran out (device status) */
  CATTN_ERR_TOO_LARGE = 5    /* shape needs more than attn_bwd_noalloc's scratch */
} cattn_status;

/* Forward pass: o = softmax(scale*q k^T + causal mask) v and its
 * log-sum-exp.  Definition as above ("nanoGPT: a real GPT in two 300-line
 * files", section 2, the written-out attention).
 *   q, k, v : in,  bf16 (B,H,T,D)
 *   scale   : softmax temperature, finite and > 0 (nanoGPT uses 1/sqrt(D))
 *   o       : out, bf16 (B,H,T,D), round-to-nearest-even
 *   lse     : out, fp32 (B,H,T), natural log
 * Errors: CATTN_ERR_INVALID_ARG (null/misaligned pointer, negative or too
 * large B, H, T, non-finite or non-positive scale), CATTN_ERR_UNSUPPORTED
 * (D, or a device other than sm_100), CATTN_ERR_CUDA. */
CATTN_API cattn_status attn_fwd(const void* q, const void* k, const void* v, float scale,
                      int B, int H, int T, int D,
                      void* o, float* lse, void* stream);

/* attn_fwd that can also write the rounding residual of its output:
 *   o_lo : out, bf16 (B,H,T,D) or NULL; o_lo = bf16(O - o) where O is the
 *          fp32 result before rounding and o = bf16(O) is the output above.
 * o + o_lo carries O to about 16 significant bits.  Handing o_lo to
 * attn_bwd_ex makes the backward's row term Delta = rowsum(dO * O) exact to
 * fp32 rounding instead of inheriting o's bf16 rounding (which, on long
 * sequences with peaked softmax, is the largest error in dQ and dK).
 * With o_lo == NULL this is exactly attn_fwd.  Errors as attn_fwd; o_lo
 * must be 16-byte aligned. */
CATTN_API cattn_status attn_fwd_ex(const void* q, const void* k, const void* v, float scale,
                                   int B, int H, int T, int D, void* o, float* lse, void* o_lo,
                                   void* stream);

/* Bytes of device workspace attn_bwd needs for this shape (0 on bad
 * arguments).  Layout: the call's status words (offset 0: CATTN_OK or the
 * first error a kernel of the call recorded; offset 4: where), then an
 * fp32 dQ accumulator of B*H*T*D floats and fp32 Delta and scaled-LSE
 * vectors of B*H*roundup(T,128) floats each; each part 256-byte aligned.
 * Only the status words are part of the interface (see
 * cattn_last_device_status). */
CATTN_API size_t attn_bwd_workspace_bytes(int B, int H, int T, int D);

/* Backward preprocess on its own: delta_i = sum_d dout_id * o_id (fp32),
 * the row term of the softmax Jacobian.  It follows from the definition
 * above by the chain rule (the pages leave the gradient to autograd:
 * "nanoGPT: a real GPT in two 300-line files", section 1, "Autograd does
 * the calculus").
 *   o, dout : in,  bf16 (B,H,T,D)
 *   delta   : out, fp32 (B,H,T)
 * Errors as attn_fwd. */
CATTN_API cattn_status attn_bwd_preprocess(const void* o, const void* dout,
                                 int B, int H, int T, int D,
                                 float* delta, void* stream);

/* Backward pass of a scalar loss L with dL/dO = dout:
 *   dV = P^T dO;  dP = dO V^T;  Delta = rowsum(dO * O);
 *   dS = P * (dP - Delta);  dQ = scale dS K;  dK = scale dS^T Q
 * P is recomputed from q, k and lse per key tile (never stored).  P
 * enters the dV product as a bf16 hi/lo pair (about 16 significant bits;
 * with P alone in bf16, dV missed the 2e-2 tolerance), dS enters the dK and
 * dQ products in bf16 (attn_bwd_ex with o_lo, or fp32 gradients, give dS a
 * hi/lo pair too); Delta is computed from the bf16 o given here (use
 * attn_bwd_ex with the forward's o_lo for an exact Delta).
 *   q, k, v, o, dout : in, bf16 (B,H,T,D); o and lse as produced by attn_fwd
 *   lse              : in, fp32 (B,H,T)
 *   dq, dk, dv       : out, bf16 (B,H,T,D)
 *   workspace        : caller-owned device scratch of at least
 *                      attn_bwd_workspace_bytes(B,H,T,D) bytes, 256-byte
 *                      aligned; overwritten; no contents needed on entry
 * Calls that share a workspace must not overlap on the GPU.
 * Errors as attn_fwd, plus CATTN_ERR_INVALID_ARG for a small or
 * misaligned workspace. */
CATTN_API cattn_status attn_bwd(const void* q, const void* k, const void* v,
                      const void* o, const float* lse, const void* dout,
                      float scale, int B, int H, int T, int D,
                      void* dq, void* dk, void* dv,
                      void* workspace, size_t workspace_bytes, void* stream);

/* Element types of gradient outputs (attn_bwd_ex). */
enum { CATTN_DTYPE_BF16 = 0, CATTN_DTYPE_F32 = 1 };

/* attn_bwd with two options:
 *   o_lo       : the forward's residual (see attn_fwd_ex) or NULL; with it
 *                Delta is computed from o + o_lo.
 *   grad_dtype : CATTN_DTYPE_BF16 (dq, dk, dv as in attn_bwd) or
 *                CATTN_DTYPE_F32: dq, dk, dv are fp32 (B,H,T,D), written
 *                without the final bf16 rounding (whose half-ulp alone is
 *                2^-8 |x|, 0.03 for gradients of magnitude 8..16).
 * o_lo == NULL with CATTN_DTYPE_BF16 is exactly attn_bwd.  Errors as
 * attn_bwd, plus CATTN_ERR_INVALID_ARG for an unknown grad_dtype. */
CATTN_API cattn_status attn_bwd_ex(const void* q, const void* k, const void* v, const void* o,
                                   const void* o_lo, const float* lse, const void* dout,
                                   float scale, int B, int H, int T, int D, void* dq, void* dk,
                                   void* dv, int grad_dtype, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* Strided tensors.
 *
 * The pages build q, k and v by splitting one projection of shape
 * (B, T, 3C) and reshaping each part to (B, T, H, D) before moving the head
 * axis forward ("nanoGPT: a real GPT in two 300-line files", section 2,
 * CausalSelfAttention: c_attn, then the heads are glued back together into
 * (B, T, C) after attention).  The _strided calls read and write such
 * views in place, with no transposes: each (B, H, T, D) operand is given by
 * its base pointer and its element strides.
 *
 *   cattn_layout { b, h, t }: element strides of the batch, head and
 *   position axes.  The d axis has stride 1.  Each stride must be a
 *   positive multiple of 8 elements (16 bytes for bf16; rows then start on
 *   16-byte boundaries) and below 2^38.  The contiguous (B, H, T, D)
 *   layout is { H*T*D, T*D, D }.  For the c_attn split, q = base,
 *   k = base + C, v = base + 2C, each with { T*3C, D, 3C }.
 *   Output (B, T, H*D) is { T*C, D, C }.
 *
 * LSE stays a contiguous (B, H, T) fp32 vector; o_lo (if given) shares o's
 * layout.  Inputs may overlap one another (q, k, v in one buffer).  Outputs
 * must not overlap each other or any input: they would race.  No output
 * may overlap itself either, and that is checked: taking the axes of
 * extent > 1 in increasing stride order (d first, stride 1, extent D),
 * each stride must be at least the span of the axes before it (the
 * contiguous layout, padded rows and the (B, T, C) output all pass).
 * Errors: as the contiguous calls, plus CATTN_ERR_INVALID_ARG for a stride
 * outside these limits or a self-overlapping output layout. */
typedef struct { long long b, h, t; } cattn_layout;

/* attn_fwd_ex with strided q, k, v and o (o_lo uses o's layout). */
CATTN_API cattn_status attn_fwd_strided(const void* q, cattn_layout lq, const void* k,
                                        cattn_layout lk, const void* v, cattn_layout lv,
                                        float scale, int B, int H, int T, int D, void* o,
                                        cattn_layout lo, float* lse, void* o_lo, void* stream);

/* attn_bwd_ex with strided q, k, v, o (and o_lo), dout, dq, dk, dv.  dq,
 * dk and dv may be the three parts of one (B, T, 3C) gradient buffer, the
 * layout the c_attn backward wants.  With CATTN_DTYPE_F32 the strides count
 * fp32 elements of dq, dk, dv. */
CATTN_API cattn_status attn_bwd_strided(const void* q, cattn_layout lq, const void* k,
                                        cattn_layout lk, const void* v, cattn_layout lv,
                                        const void* o, cattn_layout lo, const void* o_lo,
                                        const float* lse, const void* dout, cattn_layout ldo,
                                        float scale, int B, int H, int T, int D, void* dq,
                                        cattn_layout ldq, void* dk, cattn_layout ldk, void* dv,
                                        cattn_layout ldv, int grad_dtype, void* workspace,
                                        size_t workspace_bytes, void* stream);

/* Attention dropout.
 *
 * While training, the pages' CausalSelfAttention passes its dropout rate to
 * the fused attention ("nanoGPT: a real GPT in two 300-line files",
 * section 2, model.py; 0.2 for the Shakespeare model in section 3).  It is
 * inverted dropout on the attention probabilities after the softmax:
 *
 *   P~ = P * M / (1 - p),  O = P~ V,  M_ij kept with probability 1 - p,
 *
 * LSE is that of the undropped scores, and the backward holds M fixed:
 * dV = P~^T dO, dP = (dO V^T) * M / (1 - p), dS = P * (dP - Delta).
 *
 * M comes from Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random
 * numbers: as easy as 1, 2, 3", SC 2011), key = (seed low 32 bits, seed
 * high 32 bits).  Element (b, h, i, j) (query i, key j) uses the block with
 * counter (j >> 4, i, b*H + h, offset), byte j & 3 (bits 8 (j & 3) ..
 * 8 (j & 3) + 7) of word (j & 15) >> 2; it is dropped iff that byte is
 * below t = round(p * 256) (t at most 255), and kept entries are scaled by
 * 256 / (256 - t).  So the drop probability is t / 256 (p to within 2^-9)
 * and E[P~] = P exactly.  The mask depends only on (seed, offset,
 * b*H + h, i, j): the forward and backward of one step must get the same
 * seed and offset; use another offset (or seed) for every call that wants a
 * fresh mask (each layer, each step).
 *
 * dropout = NULL or p with t = 0 runs the calls without dropout (same
 * results as the _strided calls).  Errors: CATTN_ERR_INVALID_ARG for p
 * outside [0, 1) (NaN included) or a mask not 16-byte aligned, otherwise as
 * the _strided calls.  The Delta = rowsum(dO * O) of the backward holds
 * with dropout too.
 *
 * mask (optional, NULL to draw the bits in both calls): device memory of
 * attn_dropout_mask_bytes(B, H, T) bytes, 16-byte aligned.  attn_fwd_dropout
 * then also stores its keep bits there (1 bit per element of every 128 x 128
 * tile on or below the diagonal, 2 KB per tile, in the order the backward
 * reads them), and attn_bwd_dropout given the same mask reads them instead
 * of running the generator again (the generator is most of the backward's
 * dropout cost).  The results are bit-identical either way.  The caller
 * owns the buffer; its contents are valid for the backward of the forward
 * call that wrote them (same q/k/v shape, p, seed and offset), and nothing
 * checks that: a mask from another call gives wrong gradients. */
typedef struct {
  float p;                 /* drop probability, 0 <= p < 1 */
  unsigned long long seed; /* generator key */
  unsigned int offset;     /* counter word 3 */
  void* mask;              /* keep-bit cache between forward and backward, or NULL */
} cattn_dropout;

/* Bytes of a dropout keep-bit cache for B x H heads of T positions:
 * B * H * n (n + 1) / 2 * 2048 with n = ceil(T / 128); 0 for an empty or
 * invalid shape. */
CATTN_API size_t attn_dropout_mask_bytes(int B, int H, int T);

/* attn_fwd_strided with attention dropout. */
CATTN_API cattn_status attn_fwd_dropout(const void* q, cattn_layout lq, const void* k,
                                        cattn_layout lk, const void* v, cattn_layout lv,
                                        float scale, int B, int H, int T, int D,
                                        const cattn_dropout* dropout, void* o, cattn_layout lo,
                                        float* lse, void* o_lo, void* stream);

/* attn_bwd_strided with attention dropout (the forward's dropout argument). */
CATTN_API cattn_status attn_bwd_dropout(const void* q, cattn_layout lq, const void* k,
                                        cattn_layout lk, const void* v, cattn_layout lv,
                                        const void* o, cattn_layout lo, const void* o_lo,
                                        const float* lse, const void* dout, cattn_layout ldo,
                                        float scale, int B, int H, int T, int D,
                                        const cattn_dropout* dropout, void* dq, cattn_layout ldq,
                                        void* dk, cattn_layout ldk, void* dv, cattn_layout ldv,
                                        int grad_dtype, void* workspace, size_t workspace_bytes,
                                        void* stream);

/* Decode attention over a key/value cache.
 *
 * generate() in "nanoGPT: a real GPT in two 300-line files" (section 2,
 * "How the code works") runs the model once per new token; with a
 * key/value cache (as nanochat's inference does, "Karpathy's nano lineage:
 * nanoGPT, llm.c, and nanochat") a step needs causal attention only for the
 * Tq newest positions.  attn_decode computes it for query rows at positions
 * L - Tq .. L - 1 of a sequence whose first L keys and values are in k and
 * v: row r sees keys 0 .. L - Tq + r.  The result is exactly the last Tq
 * rows of attn_fwd over the whole sequence (up to rounding).
 *
 *   q      bf16 (B, H, Tq, D), layout lq
 *   k, v   bf16 (B, H, >= L, D), layouts lk, lv (rows beyond L are not
 *          read; a (B, Tmax, H, D) cache is { Tmax*H*D, D, H*D })
 *   o      bf16 (B, H, Tq, D) out, layout lo;  lse fp32 (B, H, Tq) out,
 *          contiguous, natural log
 *   workspace, workspace_bytes  not used (attn_decode_workspace_bytes
 *          returns 0 for every shape; NULL and 0 are accepted): the CTAs
 *          that share a head form a thread-block cluster and merge their
 *          partial results in distributed shared memory
 *
 * One kernel on `stream`: the keys of each head are cut into chunks of 4 KB
 * of K (2048 / D keys) dealt to a cluster of up to 8 CTAs, four warps per
 * CTA streaming their chunks.  1 <= Tq <= L; Tq above 8 returns
 * CATTN_ERR_UNSUPPORTED (use attn_fwd for a prefill).  Layout rules as for
 * the _strided calls; B = 0 or H = 0 is a no-op. */
CATTN_API size_t attn_decode_workspace_bytes(int B, int H, int Tq, int L, int D);

CATTN_API cattn_status attn_decode(const void* q, cattn_layout lq, const void* k,
                                   cattn_layout lk, const void* v, cattn_layout lv, float scale,
                                   int B, int H, int Tq, int L, int D, void* o, cattn_layout lo,
                                   float* lse, void* workspace, size_t workspace_bytes,
                                   void* stream);

/* Backward pass for callers that cannot allocate device memory.
 *
 * Same computation, arguments and results as attn_bwd, minus the workspace:
 * its scratch (the fp32 dQ accumulator and the per-row LSE and Delta
 * vectors) lives in one fixed array of CATTN_NOALLOC_SCRATCH_BYTES inside
 * the library, which every GPU that loads the library holds until the
 * process exits.  Some callers have no way to allocate: code hosted by a
 * runtime that owns all device memory and hands a plugin only its input
 * and output buffers, or latency-critical code that must not call
 * cudaMalloc / cudaFree in steady state because those calls can
 * synchronize the device.  This call allocates nothing and calls no
 * allocating routine.
 *
 * Limits and sharing:
 *  - shapes whose attn_bwd_workspace_bytes(B,H,T,D) exceeds
 *    CATTN_NOALLOC_SCRATCH_BYTES are refused with CATTN_ERR_TOO_LARGE
 *    before anything launches (the GPT-2 124M and 1558M layers fit; the
 *    T = 8192, D = 128 case does not);
 *  - every call on a device uses the same array: calls that may overlap on
 *    the GPU (different streams, or other threads) race and give wrong
 *    results; serialise them.  Each call clears and rewrites what it needs,
 *    so contents left by an earlier call do not matter;
 *  - the first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and caches it; make
 *    that first call before any stream capture.
 * The pages have no counterpart of this call: it exists for callers of
 * this library that cannot allocate.
 * Errors as attn_bwd, plus CATTN_ERR_TOO_LARGE. */
#define CATTN_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
CATTN_API cattn_status attn_bwd_noalloc(const void* q, const void* k, const void* v,
                                        const void* o, const float* lse, const void* dout,
                                        float scale, int B, int H, int T, int D, void* dq,
                                        void* dk, void* dv, void* stream);

/* Library-global device status word: CATTN_OK, or the first
 * CATTN_ERR_TIMEOUT recorded by a kernel since the last clear.  Reads it
 * synchronously (waits for all work on `stream`); clears it when `clear`
 * is non-zero.  Every kernel records here, whatever its stream: this is
 * the process-wide record, and the only one a forward call has. */
CATTN_API cattn_status cattn_get_device_status(int clear, void* stream);

/* Status of the last backward call that used `workspace` (attn_bwd and
 * its _ex/_strided/_dropout forms): CATTN_OK, or the first error one of
 * its kernels recorded (CATTN_ERR_TIMEOUT from the hang guard,
 * CATTN_ERR_UNSUPPORTED for a launch the kernel could not honour).  The
 * call's first kernel clears the words, so each call starts clean and the
 * record is that call's alone; two streams with their own workspaces never
 * see each other's failures.  Waits for all work on `stream` (the stream
 * the backward ran on), then reads the word.
 *   workspace : the call's workspace (device pointer, 256-byte aligned)
 * Errors: CATTN_ERR_INVALID_ARG for a null or misaligned pointer,
 * CATTN_ERR_CUDA if the wait or the read fails.  The word lives at offset 0
 * of the workspace whatever the shape.  ("nanoGPT: a real GPT in two
 * 300-line files" has no counterpart: PyTorch reports kernel failures
 * through its own CUDA error state.) */
CATTN_API cattn_status cattn_last_device_status(void* workspace, void* stream);

/* Time limit of every mbarrier wait inside the kernels (the hang guard), in
 * microseconds.  0 restores the default of 2 s.  Process-global; affects
 * launches made after the call.  A wait that runs out records
 * CATTN_ERR_TIMEOUT in the device status word, and its CTA skips all later
 * waits, drains the copies and MMAs it has in flight, frees its tensor
 * memory and exits (outputs are then undefined). */
CATTN_API void cattn_set_wait_timeout_us(uint32_t us);

/* Self-test of the hang guard: clears the status word, launches one tiny
 * kernel that waits on an mbarrier that nothing ever arrives on, with a
 * limit of `timeout_us`, and returns the device status that kernel recorded
 * (CATTN_ERR_TIMEOUT expected), clearing it again.  Faults nothing; the
 * CUDA context stays usable.  Synchronises `stream`. */
CATTN_API cattn_status cattn_selftest_wait_timeout(uint32_t timeout_us, void* stream);

/* The same self-test recording into a backward workspace's status words:
 * clears them, runs the waiting kernel on `stream` with `workspace` as its
 * call's record, and returns cattn_last_device_status(workspace, stream)
 * (CATTN_ERR_TIMEOUT expected).  The workspace keeps that record until a
 * backward call reuses it.  The global word is left as it was found if it
 * was clear before.  Synchronises `stream`.  Errors as
 * cattn_last_device_status. */
CATTN_API cattn_status cattn_selftest_wait_timeout_ws(uint32_t timeout_us, void* workspace,
                                                      void* stream);

/* Kernel timer (benchmarking aid).  While enabled, every kernel this
 * library launches is bracketed by two CUDA events recorded on its own
 * launching stream.  cattn_timing_read() waits for the recorded events and
 * returns, per kernel, the summed device time in ms and the launch count,
 * then forgets them.  Kernel index: 0 forward, 1 backward preprocess,
 * 2 backward main, 3 dQ convert, 4 decode (its two kernels together).
 * n = length of both output arrays (indices >= n are dropped).  Not
 * for use while a stream is being captured into a CUDA graph. */
CATTN_API void cattn_timing_enable(int enable);
CATTN_API cattn_status cattn_timing_read(float* total_ms, int* launches, int n);

/* Human-readable name of a status code (static string). */
CATTN_API const char* cattn_status_string(cattn_status s);

/* Code of the CUDA failure behind the last CATTN_ERR_CUDA returned to this
 * host thread: a cudaError_t, or 10000 + CUresult for a failed tensor-map
 * encoding; 0 if none. */
CATTN_API int cattn_last_cuda_error(void);

/* Library version, major*10000 + minor*100 + patch. */
CATTN_API int cattn_version(void);

/* How the persistent forward (kind 0) or backward (kind 1) grid of G CTAs
 * deals its work items for B*H = BH heads of n_tiles 128-row tiles
 * (diagnostic; host only, no device access).  The items are numbered
 * longest first: the forward's item u is the query-tile pair
 * c = n_pairs - 1 - u / BH (n_pairs = (n_tiles + 1) / 2), the backward's the
 * key tile u / BH, both of head u % BH.  CTA b takes one item per pass;
 * pass k deals items k*G .. k*G + G-1.  For k < the returned count,
 * codes[k] gives the pass's direction (bit 15) and rotation r (bits 0..14):
 * item k*G + j goes to CTA (r + j) mod G, or (r - j) mod G with the
 * direction bit set.  Later passes alternate: item k*G + b (k even) or
 * k*G + G-1-b (k odd) to CTA b.  The library plans the forward's codes
 * once per shape so that the CTAs' loads (an item's key tiles) stay close
 * to even; the backward's passes always alternate (count 0).  Writes at
 * most max_codes codes; returns their count, or -1 for kind not 0 or 1,
 * BH < 1, n_tiles < 1 or G < 1. */
CATTN_API int cattn_plan_passes(int kind, int BH, int n_tiles, int G, uint16_t* codes,
                                int max_codes);

#ifdef __cplusplus
}
#endif

#endif /* CATTN_H */
