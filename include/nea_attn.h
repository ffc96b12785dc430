/*
 * nea_attn.h -- C ABI of the B200 (sm_100a) causal grouped-query attention
 * library: forward and backward of softmax attention with rotary position
 * embeddings on queries and keys.
 *
 * Operation (the tiled FlashAttention of a bias-free decoder-only
 * transformer: "NanoEuler" write-up, aimsg.uk, section 4 "GPU version",
 * FlashAttention bullet -- tiled, online softmax, the T x T matrix never kept
 * in memory; section 2 "Model components": RoPE on queries and keys, GQA,
 * no bias terms; "Tiny Hackable CUDA LM", aimsg.uk, section 1: causal
 * scaled dot-product attention):
 *
 *   q'_t = R_t q_t,  k'_t = R_t k_t   (R_t turns each interleaved pair
 *                                      (x[2i], x[2i+1]) by t * base^(-2i/D);
 *                                      t = 0 .. T-1; V is not rotated)
 *   s_ij = q'_i . k'_j / sqrt(D),     masked for j > i when causal
 *   LSE_i = ln sum_j exp(s_ij),  P_ij = exp(s_ij - LSE_i),  O_i = sum_j P_ij v_j
 *
 * Query head h reads key/value head floor(h / (Hq / Hkv)).
 *
 * Layouts (row-major, contiguous, element type given by `dtype`):
 *   Q, O, dO, dQ : [B][T][Hq][D]
 *   K, V, dK, dV : [B][T][Hkv][D]
 *   LSE          : [B][Hq][T], always float32
 *
 * Ownership: every pointer is a device pointer owned by the caller; the
 * library never frees or retains them.  The library keeps, per device, a
 * cached workspace (the rotary cos/sin tables, the backward's per-row terms
 * and the operand prologue's output), allocated on first use and
 * grown only when a call needs more; steady-state calls allocate nothing.
 *
 * Streams: work is enqueued on `stream` (a cudaStream_t, NULL for the legacy
 * default stream) and the call returns without synchronising.  Calls on one
 * device share its workspace, so calls on different streams must not overlap
 * in time.  Device-side wait limits are reported asynchronously: see
 * nea_device_status().  The training-path kernels are launched with
 * programmatic stream serialization: a kernel may begin its set-up while the
 * kernel before it in the stream drains, but it touches no global memory
 * until that kernel has completed, so stream order holds for every buffer
 * (the caller's kernels included).
 *
 * Errors: a call returns NEA_OK or one of the codes below; on NEA_ERR_ARG
 * nothing is launched and no output is touched.  Kernels never trap.
 */
#ifndef NEA_ATTN_H
#define NEA_ATTN_H

#ifdef __cplusplus
extern "C" {
#endif

/* Element type of Q, K, V, O, dO, dQ, dK, dV. */
typedef enum {
  NEA_F32 = 0,  /* float32 storage; every contraction in split bf16 (see below) */
  NEA_BF16 = 1  /* bfloat16 storage; bf16 tensor-core operands, fp32 accumulation */
} nea_dtype;

enum {
  NEA_OK = 0,
  NEA_ERR_ARG = 1,         /* invalid pointer, shape, alignment or dtype */
  NEA_ERR_CUDA = 2,        /* a CUDA runtime call or kernel launch failed */
  NEA_ERR_TIMEOUT = 3,     /* a kernel gave up a bounded device-side wait */
  NEA_ERR_UNSUPPORTED = 4, /* current device is not sm_100 */
  NEA_ERR_NOMEM = 5,       /* workspace allocation failed */
  NEA_ERR_SCRATCH_LIMIT = 6 /* problem too large for nea_attn_bwd_noalloc's fixed scratch */
};

/*
 * Forward.  Writes O and LSE.
 *
 *   Q, K, V     inputs, see layouts above; 16-byte aligned
 *   O           output, same shape and dtype as Q
 *   LSE         output, float32 [B][Hq][T], natural-log log-sum-exp of the
 *               scaled, masked scores of each query row
 *   B, T        batch and sequence length, >= 0 (B*T == 0 is a no-op)
 *   Hq, Hkv     query and key/value heads, Hq % Hkv == 0
 *   D           head dimension, 32 or 64; also 128 with NEA_BF16 (forward, backward
 *               and the save-for-backward pair; float32 storage and
 *               nea_attn_bwd_noalloc return NEA_ERR_ARG for D = 128)
 *   dtype       NEA_F32 or NEA_BF16
 *   rope_base   rotary base (10000 for the workloads here); <= 0 disables
 *               the rotation
 *   causal      1: key j visible to query i iff j <= i; 0: all keys visible
 *   stream      cudaStream_t to enqueue on
 *
 * An operand prologue kernel first applies the rotation to Q and K, once per
 * element, into the workspace.  NEA_BF16: the rotated copies (rounded to
 * bf16) feed plain bf16 tensor-core products with fp32 accumulation.
 * NEA_F32: the prologue writes Q, K, V as bf16 high and low planes; each
 * score and output contraction is formed from them as hi*hi + hi*lo + lo*hi
 * (fp32 accumulation), about 2^-16 relative per product.
 */
int nea_attn_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int T, int Hq,
                 int Hkv, int D, int dtype, float rope_base, int causal, void* stream);

/*
 * Backward.  Given the forward's inputs, its outputs O and LSE, and the
 * upstream gradient dO, writes dQ, dK, dV: gradients with respect to the
 * un-rotated Q and K and to V, with dK and dV summed over the query heads of
 * each group.  Arguments as for nea_attn_fwd; dQ has the shape of Q, dK and
 * dV the shape of K.  O and LSE must be the forward's results for the same
 * Q, K, V, rope_base and causal.
 *
 * Runs on `stream`: the operand prologue (NEA_F32: bf16 hi/lo planes of the
 * rotated Q and K and of V, dO; NEA_BF16: rotated copies of Q and K, none
 * when the rotation is off), which in the same launch writes the row terms
 * -LSE*log2(e) and D_i = sum_d dO_id O_id; one gradient kernel whose CTAs
 * run dK/dV units (one per key tile and kv head, looping over the query heads
 * of the group) and dQ units (one per query tile and head); both recompute P
 * from LSE.
 *
 * NEA_F32: all five products (S, dP = dO V^T, dV, dK, dQ) use split bf16 as
 * in the forward -- each operand as bf16 high and low parts, each product as
 * hi*hi + hi*lo + lo*hi with fp32 accumulation (about 2^-16 relative per
 * product, finer than TF32); P and dS are split by the kernel before their
 * products.
 */
int nea_attn_bwd(const void* Q, const void* K, const void* V, const void* O, const float* LSE, const void* dO,
                 void* dQ, void* dK, void* dV, int B, int T, int Hq, int Hkv, int D, int dtype, float rope_base,
                 int causal, void* stream);

/*
 * Save-for-backward pair.  The forward's operand prologue (rotated Q and K;
 * for NEA_F32 also the bf16 hi/lo planes of Q, K and V) produces exactly the
 * operands the backward needs again.  nea_attn_fwd_save writes them into a
 * caller-owned buffer `saved` instead of the library workspace, and
 * nea_attn_bwd_saved reads them from there, so the backward's prologue only
 * converts dO and writes the row terms.
 *
 * nea_attn_saved_bytes: the size of `saved` for these arguments (the same for
 * either value of causal): NEA_F32 4*(B*T*(Hq + 2*Hkv)*D) bytes, each plane
 * rounded up to 256 bytes; NEA_BF16 with the rotation on, the rotated Q and K
 * (2*B*T*(Hq + Hkv)*D bytes, rounded likewise); NEA_BF16 with the rotation
 * off, 0.  Returns -1 for arguments the forward would reject.
 *
 * nea_attn_fwd_save: nea_attn_fwd with the planes written to `saved` (device
 * memory, 16-byte aligned, at least nea_attn_saved_bytes bytes, owned by the
 * caller; may be NULL when that size is 0).  O and LSE are bit-identical to
 * nea_attn_fwd's.
 *
 * nea_attn_bwd_saved: nea_attn_bwd with Q, K and V operands taken from
 * `saved`.  `saved` must hold what nea_attn_fwd_save wrote for the same Q, K,
 * V, B, T, Hq, Hkv, D, dtype and rope_base, and must not have been written
 * since; Q, K and V are still passed (and checked) but their values are not
 * read.  With those inputs dQ, dK, dV are bit-identical to nea_attn_bwd's.
 * The library cannot check the contents of `saved`: stale planes give
 * gradients of the tensors they were made from.  When the saved size is 0
 * this is nea_attn_bwd.  Errors as for nea_attn_bwd, plus NEA_ERR_ARG for a
 * NULL or unaligned `saved` of nonzero size.
 */
long long nea_attn_saved_bytes(int B, int T, int Hq, int Hkv, int D, int dtype, float rope_base);
int nea_attn_fwd_save(const void* Q, const void* K, const void* V, void* O, float* LSE, void* saved, int B, int T,
                      int Hq, int Hkv, int D, int dtype, float rope_base, int causal, void* stream);
int nea_attn_bwd_saved(const void* Q, const void* K, const void* V, const void* O, const float* LSE, const void* dO,
                       const void* saved, void* dQ, void* dK, void* dV, int B, int T, int Hq, int Hkv, int D,
                       int dtype, float rope_base, int causal, void* stream);

/*
 * Decoder-block steps beside the attention ("NanoEuler" write-up, aimsg.uk,
 * section 1 "Architecture design" and section 2 "Model components": a
 * pre-norm block x <- x + Attn(RMSNorm(x)), RMSNorm without bias, no bias in
 * any projection):
 *
 *   rstd_m = (mean_c x_mc^2 + 1e-5)^(-1/2),  y = x rstd g
 *   q = y Wq,  k = y Wk,  v = y Wv           (the attention's inputs, un-rotated)
 *   h = x + o Wo                             (o: the attention's output)
 *
 * Layouts (row-major, contiguous, element type `dtype` as for the attention;
 * M = B*T tokens):
 *   x, h, dx, dh : [M][C];   g, dg : [C]
 *   Wq, dWq      : [C][Hq*D];   Wk, Wv, dWk, dWv : [C][Hkv*D]
 *   Wo, dWo      : [Hq*D][C]
 *   q, dq, o, do : [M][Hq*D] (= [B][T][Hq][D]);  k, v, dk, dv : [M][Hkv*D]
 * C and Hkv*D must be multiples of 64; D a multiple of 8; Hq % Hkv == 0.
 * Every product runs on the library's tcgen05 GEMM: bf16 operands with fp32
 * accumulation for NEA_BF16; for NEA_F32 each operand as bf16 hi and lo
 * planes and each product as hi*hi + hi*lo + lo*hi (as in the attention).
 * The steps keep a per-device workspace of their own (operand planes, the
 * norm's fp32 input gradient), grown when a call needs more.  Errors and
 * streams as for the attention; nothing is launched on NEA_ERR_ARG.
 *
 * nea_block_qkv_fwd: q, k, v from x (the norm is applied inside).
 * nea_block_qkv_bwd: from the forward's inputs and the upstream gradients dq,
 *   dk, dv (gradients of the un-rotated q, k, v -- nea_attn_bwd's outputs):
 *   dWq = y^T dq (likewise dWk, dWv), dy = dq Wq^T + dk Wk^T + dv Wv^T,
 *   dx = rstd g dy - x rstd^3 / C sum_c (g dy)_c x_c, plus `dres` when it is
 *   not NULL (the residual branch's gradient, dh), and dg = sum_m dy x rstd.
 *   The norm is recomputed from x.
 * nea_block_out_fwd: h = x + o Wo.
 * nea_block_out_bwd: do = dh Wo^T and dWo = o^T dh (the residual's gradient
 *   is dh itself).
 */
int nea_block_qkv_fwd(const void* x, const void* g, const void* Wq, const void* Wk, const void* Wv, void* q, void* k,
                      void* v, int M, int C, int Hq, int Hkv, int D, int dtype, void* stream);
int nea_block_qkv_bwd(const void* x, const void* g, const void* Wq, const void* Wk, const void* Wv, const void* dq,
                      const void* dk, const void* dv, const void* dres, void* dx, void* dg, void* dWq, void* dWk,
                      void* dWv, int M, int C, int Hq, int Hkv, int D, int dtype, void* stream);
int nea_block_out_fwd(const void* x, const void* o, const void* Wo, void* h, int M, int C, int Hq, int D, int dtype,
                      void* stream);
int nea_block_out_bwd(const void* o, const void* Wo, const void* dh, void* do_, void* dWo, int M, int C, int Hq,
                      int D, int dtype, void* stream);

/*
 * The block's feed-forward half, a pre-norm SwiGLU with its residual add
 * ("NanoEuler" write-up, section 2 "Model components", SwiGLU feed-forward:
 * down(silu(gate(x)) * up(x)) with silu(z) = z / (1 + e^-z)):
 *
 *   y = x rstd g (the RMSNorm above),  a = y Wg,  b = y Wu,
 *   h = x + (silu(a) * b) Wd             (* elementwise)
 *
 * Layouts (row-major, contiguous, element type `dtype`; M = B*T tokens):
 *   x, h, dx, dh : [M][C];   g, dg : [C];   a, b : [M][F]
 *   Wg, Wu, dWg, dWu : [C][F];   Wd, dWd : [F][C]
 * C and F must be multiples of 64, C <= 4096.  Products, precision,
 * workspace, errors and streams as for the steps above.
 *
 * nea_block_ffn_fwd: h from x; the gate and up pre-activations a and b are
 *   written to the caller's buffers for the backward (save for backward;
 *   either may be NULL when no backward follows).  silu(a) b is formed in
 *   the epilogue of the gate/up product and never stored in the storage
 *   type: the down product reads it in fp32 precision (NEA_F32) or bf16.
 * nea_block_ffn_bwd: from the forward's inputs, its a and b, and the
 *   upstream gradient dh: with s = sigmoid(a), dact = dh Wd^T,
 *   da = dact b s (1 + a (1 - s)), db = dact silu(a),
 *   dWd = (silu(a) b)^T dh,  dWg = y^T da,  dWu = y^T db,
 *   dy = da Wg^T + db Wu^T, and dx, dg from dy through the norm as in
 *   nea_block_qkv_bwd, dx including the residual's dh.  The norm is
 *   recomputed from x.
 */
int nea_block_ffn_fwd(const void* x, const void* g, const void* Wg, const void* Wu, const void* Wd, void* h, void* a,
                      void* b, int M, int C, int F, int dtype, void* stream);
int nea_block_ffn_bwd(const void* x, const void* g, const void* Wg, const void* Wu, const void* Wd, const void* a,
                      const void* b, const void* dh, void* dx, void* dg, void* dWg, void* dWu, void* dWd, int M, int C,
                      int F, int dtype, void* stream);

/*
 * Synchronises `stream`, then reads and clears the device status words of the
 * current device: the one the regular entry points write and the one inside
 * the fixed scratch of nea_attn_bwd_noalloc.  Returns NEA_OK, NEA_ERR_TIMEOUT
 * when a kernel since the last call abandoned a bounded wait (its outputs
 * are then undefined), NEA_ERR_ARG when a decode call met a cache length
 * outside [0, Tc], or NEA_ERR_CUDA when the synchronisation or the read
 * failed.  It sets up neither word (a word that was never set up reads as
 * clear), so it never allocates device memory.
 */
int nea_device_status(void* stream);

/*
 * Sets the per-wait device limit in nanoseconds for later launches on this
 * host thread (default 2e9; values < 1e6 are raised to 1e6).  Returns the
 * previous value.
 */
long long nea_set_wait_limit_ns(long long ns);

/*
 * Fault-injection hook for tests, for later launches on this host thread:
 *   flags & 1: the next forward launch withholds the query-tile arrival its
 *              MMA issuers wait for;
 *   flags & 2: the next backward launch (nea_attn_bwd or
 *              nea_attn_bwd_noalloc) withholds the resident-tile arrival of
 *              its gradient kernel.
 * Every dependent wait then runs into its limit, the kernel returns, and
 * NEA_ERR_TIMEOUT is pending for nea_device_status().  Each bit is cleared
 * by the launch it arms.
 */
void nea_debug_inject(int flags);

/*
 * Profiling hook.  `events` points at `n` cudaEvent_t handles owned by the
 * caller (NULL / 0 disables).  While set, later calls on this host thread
 * record them on their stream at kernel boundaries:
 *   nea_attn_fwd: events[0] before the operand prologue, events[6] after it
 *                 (before the forward kernel), events[1] after the forward
 *                 kernel;
 *   nea_attn_bwd: events[2] before the operand prologue (which also writes
 *                 the row terms), events[3] after it, events[4] and events[5]
 *                 after the gradient kernel.
 * Indices >= n are skipped.  The array must stay valid while set.  An event
 * between two kernels stops the second from starting early, so profiled
 * calls run their kernels strictly one after the other.
 */
void nea_set_profile_events(void* const* events, int n);

/*
 * Backward without any device allocation.  The source pages have no
 * counterpart; this entry point exists for callers that must not call
 * cudaMalloc or cudaFree themselves or through a library -- code that runs
 * under a host-side memory manager that owns every device buffer (custom
 * allocators, pre-planned arenas, some embedded or real-time hosts), or code
 * whose allocations would synchronise or fragment the device at a bad time.
 *
 * Same arguments, layouts and results as nea_attn_bwd.  The caller passes all
 * inputs and outputs; everything else the backward needs (the per-row terms
 * -LSE*log2(e) and D_i = sum_d dO_id O_id, the rotary cos/sin table -- built
 * by the same device kernel as the regular entry points' table, so the two
 * are bit-identical -- a device status word and the operand prologue's
 * output: for NEA_F32 the bf16 hi/lo planes of Q, K, V, dO, for NEA_BF16 with
 * the rotation on the rotated copies of Q and K) lives in one fixed array of
 * 4 MiB compiled into the library: every GPU that loads the library keeps it
 * until the process exits.  With Tp = 128*ceil(T/128), a call needs about
 * 256 + 8*B*Hq*Tp bytes of it, plus 4*T*D bytes with the rotation on, plus
 * 8*B*T*(Hq + Hkv)*D bytes for NEA_F32 or, with the rotation on,
 * 2*B*T*(Hq + Hkv)*D bytes for NEA_BF16 (each part rounded up to 256
 * bytes); larger problems return NEA_ERR_SCRATCH_LIMIT before anything is
 * launched.
 *
 * The first call on a device does a one-time set-up with that device
 * current (it looks up the array's device address and sets kernel
 * attributes); make that first call before any stream capture.  All calls
 * share the one array and it keeps the last call's contents, so calls whose
 * work may overlap on the GPU (different streams without ordering, or
 * several host threads) race and must be serialised by the caller.  A
 * device-side wait that runs into its limit sets the array's status word
 * (outputs are then undefined); nea_device_status() reports it as
 * NEA_ERR_TIMEOUT and clears it, allocating nothing.
 */
int nea_attn_bwd_noalloc(const void* Q, const void* K, const void* V, const void* O, const float* LSE,
                         const void* dO, void* dQ, void* dK, void* dV, int B, int T, int Hq, int Hkv, int D,
                         int dtype, float rope_base, int causal, void* stream);

/*
 * Decode: attention of one new query per sequence over a key/value cache,
 * the generation path of the same causal attention ("NanoEuler" write-up,
 * aimsg.uk, section 1, head-0 generation; RoPE on the query at its position,
 * section 2 "Model components").
 *
 *   Q      [B][Hq][D] un-rotated query of the token at position lens[b] - 1
 *   Kc     [B][Tc][Hkv][D] cached keys, already rotated at their positions
 *          (R_t k_t, the same rotation the training path applies)
 *   Vc     [B][Tc][Hkv][D] cached values
 *   lens   device int32 [B]: valid cache length of each sequence,
 *          0 <= lens[b] <= Tc; position lens[b] - 1 is the query's own
 *   O      output [B][Hq][D], same dtype as Q
 *   LSE    output float32 [B][Hq], natural-log log-sum-exp of the scores
 *   Tc     cache capacity (positions), 1 <= Tc <= 2^24
 *   Hq / Hkv <= 8; D 32, 64 or 128; dtype NEA_F32 or NEA_BF16 (all arithmetic in
 *   fp32); rope_base <= 0 disables the rotation of the query.
 *
 *   q' = R_{lens[b]-1} q, s_j = q' . k_j / sqrt(D) for j < lens[b],
 *   LSE = ln sum_j exp(s_j), O = sum_j exp(s_j - LSE) v_j;
 *   lens[b] = 0 gives O = 0 and LSE = -inf.
 *
 * Runs one kernel over 128-position pieces of the cache (the last piece of
 * each sequence and kv head to finish merges them); uses the per-device
 * workspace (B*Hq*ceil(Tc/128)*(D+2) floats and B*Hkv counters, cleared by
 * the call).
 * The lengths are read on the device: a value outside [0, Tc] is clamped and
 * reported by the next nea_device_status() as NEA_ERR_ARG.  B == 0 is a
 * no-op; argument errors return NEA_ERR_ARG with nothing launched.
 */
int nea_attn_decode(const void* Q, const void* Kc, const void* Vc, const int* lens, void* O, float* LSE, int B,
                    int Tc, int Hq, int Hkv, int D, int dtype, float rope_base, void* stream);

/* Human-readable name of a status code (static storage). */
const char* nea_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int nea_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NEA_ATTN_H */
