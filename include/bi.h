/* bi.h -- C ABI of the batch-invariant decoder library (libbi.so, sm_100a).
 *
 * Every call computes the same per-row result whatever else is in the batch:
 * the reduction order of every sum (GEMM K loop, RMSNorm, attention score
 * sum, softmax denominator, PV accumulation, LM-head logsumexp) is fixed and
 * depends neither on the number of rows, nor on how prefill is chunked, nor
 * on prefill vs decode.  This is the method of the page "Meituan bitwise
 * train/infer consistency" (root-cause list: attention score sums, softmax
 * denominators, cross-device matrix reductions and logprob accumulation;
 * scheme: fix the order of every reduce-add and share one reduction path
 * between training, Prefill and Decode; TP computed over the full K
 * dimension instead of segmented reduce-scatter).
 *
 * Conventions for every function:
 *  - extern "C", returns int status (bi_status).  On failure nothing has been
 *    launched and bi_last_error() returns a message (thread-local).
 *  - Work is enqueued on the given CUDA stream (a cudaStream_t passed as
 *    void*; NULL = legacy default stream) and runs asynchronously; a fault
 *    inside a kernel surfaces at the caller's next synchronisation.
 *  - Ownership: the caller owns EVERY device buffer (weights, KV cache,
 *    inputs, outputs, workspace).  The library never allocates or frees
 *    device memory and keeps no pointer after a call returns, except that a
 *    bi_ctx stores the caller's weight/KV pointers until bi_ctx_destroy.
 *  - Pointers marked (device) must be device-accessible; (host) are read on
 *    the host during the call only.  Layouts are row-major, contiguous unless
 *    a leading dimension is given.
 *  - bf16 = IEEE bfloat16 bit pattern (uint16); f32 = IEEE binary32.
 *  - Kernels use programmatic dependent launch: a library kernel may start
 *    while the library kernel before it on the stream is finishing.  The GEMM
 *    reads its weight w before it waits for that kernel; every other operand
 *    of every call is touched only after the wait.  So a GEMM weight must not
 *    be the output of the library call enqueued just before it (kernels of the
 *    caller's own, copies and other libraries are waited for in full).
 */
#ifndef BI_H
#define BI_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BI_OK = 0,
  BI_ERR_INVALID_ARG = 1, /* NULL pointer, negative size, inconsistent batch */
  BI_ERR_UNSUPPORTED = 2, /* shape or mode the kernels do not implement */
  BI_ERR_WORKSPACE = 3,   /* workspace NULL or smaller than *_workspace_size */
  BI_ERR_CAPACITY = 4,    /* position beyond KV capacity or RoPE table */
  BI_ERR_CUDA = 5         /* a CUDA runtime/driver call failed at launch */
} bi_status;

enum { BI_MODE_BF16 = 0, BI_MODE_LAYERCAST = 1, BI_MODE_FP32 = 2 };
/* BI_MODE_BF16: bf16 activations and KV cache, bf16 x bf16 products with fp32
 *   accumulation on tensor cores, fp32 softmax/norm arithmetic.
 * BI_MODE_LAYERCAST: the "LayerCast" scheme of "Give Me FP32 or Give Me
 *   Death?" (LayerCast section): weights stay bf16 in memory and the
 *   arithmetic is fp32; activations and KV cache are fp32.  Projections take
 *   exact fp32 products on the tensor cores (see bi_gemm); the LM head,
 *   attention and norms use fp32 FMA on the CUDA cores, with the bf16
 *   weights cast to fp32 in registers.
 * BI_MODE_FP32: full FP32 storage, the arm LayerCast is compared with in
 *   "Give Me FP32 or Give Me Death?" (LayerCast section; jiaxiangli.netlify.app
 *   write-up, section 4): the projection, embedding and LM-head weights are f32
 *   in memory (the norm gains stay bf16), activations and KV cache are f32,
 *   and every product and sum is an fp32 FMA on the CUDA cores.  A reference
 *   arm for the precision study, not a fast path. */
enum { BI_VARIANT_INVARIANT = 0, BI_VARIANT_FAST = 1 };
/* BI_VARIANT_FAST is the non-invariant comparison baseline: split-K GEMMs
 * whose split factor is chosen from the row count M and the SM count, and
 * attention whose KV split is chosen from the batch size.  Its results are
 * deterministic for a fixed shape but change with batch size.  Not a product
 * path; it exists so the cost of invariance can be measured. */
enum { BI_DTYPE_BF16 = 0, BI_DTYPE_F32 = 1 };
enum { BI_EPI_NONE = 0, BI_EPI_SWIGLU = 1, BI_EPI_ROPE_KV_APPEND = 2 };

/* Granule of the gate/up interleave used by BI_EPI_SWIGLU: the fused weight
 * holds 16 gate rows, then the 16 up rows of the same output columns, etc. */
#define BI_GU_INTERLEAVE 16
/* Absolute KV chunk size of the attention grid (positions 0..255, 256..511, ...). */
#define BI_ATTN_CHUNK 256
/* Vocabulary chunk of the LM-head partial reductions. */
#define BI_VOCAB_CHUNK 256

const char* bi_last_error(void);
int bi_version(void);
/* Device error word: kernels never trap; a bounded wait that runs out, a
 * position beyond capacity or an out-of-range id sets a bit here instead
 * (1 = wait timeout, 2 = capacity, 4 = index) and the kernel skips the access.
 * Bits 8 and up name the first wait that ran out (a site code of the kernel:
 * 0x11/0x12/0x13 GEMM ring empty/full/drain, 0x21/0x22 attention, 0x31 the
 * wait self-test; higher bits carry the kernel's configuration), 0 when none
 * did.  Every wait gives up after about 1 s of wall-clock time.
 * Synchronous read of the current device's word; reset != 0 clears it. */
int bi_device_error(unsigned* flags, int reset);
/* Failure-path check of the bounded waits, without faulting the GPU: one CTA
 * waits on a barrier that nothing completes; after about 1 s the wait gives up,
 * sets bit 1 of the device error word with site code 0x31, and the kernel
 * returns, leaving the context usable.  Asynchronous on the stream; read the
 * outcome with bi_device_error after synchronising. */
int bi_selftest_wait_timeout(void* stream);
int bi_num_sms(int device); /* SM count of a device, -1 on error */
/* Number of kernels the library has launched in this process (host-side
 * counter, incremented at every launch site; not thread-safe). */
long long bi_launch_count(void);

/* --------------------------------------------------------------- KV cache
 * k and v: [n_slots][n_layers][n_kv_heads][capacity][head_dim], dtype bf16
 * (BI_MODE_BF16) or f32 (BI_MODE_LAYERCAST).  Position p of slot s is row p. */
typedef struct {
  void* k;
  void* v;
  int n_slots, n_layers, n_kv_heads, capacity, head_dim;
  int dtype; /* BI_DTYPE_BF16 or BI_DTYPE_F32 */
} bi_kv_layout;

/* RoPE table: [max_pos][head_dim/2][2] f32 (cos, sin) of pos * theta^(-2i/d),
 * evaluated in fp64 on the host and rounded to f32.  Rotate-half pairing
 * (i, i + d/2).  table: device, caller-allocated max_pos*head_dim floats. */
int bi_rope_table_fill(float* table, int max_pos, int head_dim, double theta, void* stream);

/* ------------------------------------------------------------------ GEMM
 * y[m][n] = sum_k x[m][k] * w[n][k]   (x: [M][K] with leading dim ldx,
 *   w: bf16 [N][K] contiguous, y: [M][N] with leading dim ldy).
 * Invariant variant ("Meituan bitwise train/infer consistency": TP rewritten
 *   to full-K computation instead of segmented reduce-scatter, one reduction
 *   path shared by Prefill and Decode): each output element is accumulated in
 *   fp32 over the FULL K range by tensor-core MMA instructions of K = 16 in
 *   ascending K, the k16 steps going round-robin into KS interleaved
 *   accumulators that are added in a fixed tree at the end: KS = 4 for
 *   matrices of N <= 8192 rows, 1 for larger N divisible by 128, else 2.
 *   ((s0 + s1) + (s2 + s3), s0 + s1 or s0.)  KS is a property of the matrix,
 *   never of M: no split-K, and a row's result does not depend on the other
 *   rows of the call, nor on which tensor-core path (mma.sync for at most 32
 *   rows, tcgen05 above: the same arithmetic) runs it.
 * n_full: 0 when w is a whole weight matrix; else the output rows of the
 *   matrix that w is a contiguous row shard of (tensor parallelism), which
 *   then fixes KS, so a shard's rows are bitwise the unsharded call's.  A
 *   shard must hold whole 128/KS-row tiles (else BI_ERR_UNSUPPORTED).
 * mode BI_MODE_BF16: x is bf16.  mode BI_MODE_LAYERCAST: x is f32 and the
 *   products are fp32-exact: every x is split exactly into three bf16 parts
 *   (x = p0 + p1 + p2, 8+8+8 significant bits), each part times the bf16 w is
 *   an exact product accumulated in fp32 on the tensor cores (full K,
 *   ascending, as above), and the three sums are added as (y0 + y1) + y2
 *   before the epilogue.
 * y_dtype: BI_DTYPE_BF16 (round-to-nearest-even) or BI_DTYPE_F32.
 * epilogue BI_EPI_SWIGLU: w rows are gate/up interleaved by BI_GU_INTERLEAVE
 *   and y has N/2 columns: y = silu(gate) * up, silu(g) = g / (1 + exp(-g)).
 * epilogue BI_EPI_ROPE_KV_APPEND (BI_MODE_BF16, invariant variant only): the
 *   QKV projection of one decoder layer with rotate-half RoPE and the KV-cache
 *   append in its epilogue (the pages name the steps, not the fusion, which
 *   is this library's).  w is one layer of bi_weights.w_qkv (q and k heads in
 *   the paired row order described there), N = (Hq + 2 Hkv) * head_dim.  The
 *   f32 projection of each q and k head is rotated at pos[m] with the f32
 *   table of bi_rope_table_fill (for the pair (a, b) = (x[i], x[i + d/2]):
 *   a' = a c - b s, b' = b c + a s), then q is stored (bf16, natural element
 *   order) to epi->q_out [M][Hq * head_dim] and k, v (bf16) to the cache
 *   epi->kv at (slot[m], epi->layer, head, pos[m]).  y and ldy are unused (y
 *   may be NULL).  A row whose slot or position is out of range sets the
 *   capacity bit of the device error word and is skipped.  epi must be NULL
 *   for the other epilogues.
 * Requirements: K % 64 == 0, N % 64 == 0, ldx % 8 == 0 (16-byte rows),
 *   x, w 16-byte aligned; else BI_ERR_UNSUPPORTED.  M == 0 is a no-op
 *   (x and y may then be NULL); w NULL is BI_ERR_INVALID_ARG.
 * Workspace: bi_gemm_workspace_size() bytes (0 for the invariant bf16 mode;
 *   LayerCast needs room for the split rows and their three partial sums). */
typedef struct {
  const float* rope;      /* device RoPE table from bi_rope_table_fill */
  int rope_max_pos;       /* positions the table holds */
  void* q_out;            /* device [M][n_heads * head_dim] bf16 */
  const bi_kv_layout* kv; /* host struct; kv->k and kv->v are the device cache (bf16) */
  int layer;              /* layer of the cache the rows are appended to */
  const int32_t* slot;    /* device [M]: KV slot of each row */
  const int32_t* pos;     /* device [M]: position of each row in its slot */
  int n_heads;            /* Hq (Hkv and head_dim come from kv) */
} bi_epi_args;
size_t bi_gemm_workspace_size(int M, int N, int K, int mode, int variant);
int bi_gemm(const void* x, int ldx, const void* w, void* y, int ldy, int y_dtype, int M, int N, int K, int n_full,
            int epilogue, const bi_epi_args* epi, int mode, int variant, void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------- RMSNorm
 * Per row m (fused residual add, as in a pre-norm decoder):
 *   r'  = x + residual_in          (residual_in NULL: r' = x)
 *   residual_out = r' (rounded to the activation dtype; may alias residual_in)
 *   y   = r' / sqrt(mean(r'^2) + eps) * gamma        (activation dtype)
 *   y_f32 (optional, f32) = the same value before rounding.
 * The mean of squares is a fixed reduction tree over H (per-thread strided
 * partials, fixed shuffle tree, ascending cross-warp sum) that does not
 * depend on M ("Meituan bitwise train/infer consistency", key-practices list:
 * batch-invariant operators with one reduction order for training, Prefill
 * and Decode; the pages do not name RMSNorm, the architecture comes from the
 * model shapes of the workloads).  Activation dtype: bf16 (BI_MODE_BF16) or
 * f32 (LAYERCAST).  gamma: bf16 [H].  H % 8 == 0 and H <= 16384. */
int bi_rmsnorm(const void* x, const void* residual_in, void* residual_out, const void* gamma, void* y,
               float* y_f32, int M, int H, float eps, int mode, void* stream);

/* Rotary embedding + KV append for T tokens after the QKV projection (the
 * pages are silent on positional encoding: rotate-half RoPE of the Llama- and
 * Qwen-shaped workloads, no frequency scaling; the LayerCast and FAST paths
 * use this kernel, the bf16 invariant path the fused GEMM epilogue).
 * qkv: f32 [T][(Hq + 2*Hkv) * d] (q heads, then k heads, then v heads).
 * q_out: [T][Hq*d] activation dtype; k and v rows are written to the cache at
 * (slot[t], layer, head, pos[t]).  slot/pos: device int32 [T].
 * qk_paired != 0: each q and k head of qkv is in the paired row order of
 * bi_weights.w_qkv (below); q_out and the cache are always in natural order. */
int bi_rope_kv_append(const float* qkv, const float* rope, int rope_max_pos, void* q_out, const bi_kv_layout* kv,
                      int layer, const int32_t* slot, const int32_t* pos, int T, int Hq, int qk_paired, int mode,
                      void* stream);

/* ------------------------------------------------------------- Attention
 * For each token t and q head h (kv head h / (Hq/Hkv)): causal softmax
 * attention of q[t][h] over positions 0..pos[t] of slot[t]'s cache:
 *   s_j = scale * q . k_j,  out = sum_j softmax(s)_j v_j.
 * Fixed order ("Meituan bitwise train/infer consistency": the attention score
 * sum and softmax denominator must reduce in one order for Prefill and Decode):
 * the keys are cut on the ABSOLUTE grid of BI_ATTN_CHUNK positions; per chunk
 * the partial (max, sum of exp, sum of p*v) is formed with fixed trees; the
 * chunk partials are merged in ascending chunk order.  A query's result
 * depends only on its own q and the cache rows it reads.
 * q: [T][Hq*d], out: [T][Hq*d] (activation dtype); slot/pos: device int32 [T];
 * slot_host/pos_host: host copies (validation and work planning).  Tokens of
 * one slot that are adjacent in the batch must have consecutive positions.
 * head_dim must be 64 or 128. */
size_t bi_attention_workspace_size(int T, int Hq, int head_dim, int max_pos);
int bi_attention(const void* q, const bi_kv_layout* kv, int layer, const int32_t* slot, const int32_t* pos,
                 const int32_t* slot_host, const int32_t* pos_host, void* out, int T, int Hq, float scale, int mode,
                 int variant, void* ws, size_t ws_bytes, void* stream);

/* -------------------------------------------------------- LM-head logprob
 * For each row b of h (f32 [B][H], device):
 *   z = h . W^T (W bf16 [V][H]).  BI_MODE_BF16: h is rounded to bf16 and
 *   z is a bf16 x bf16 tensor-core product with fp32 accumulation.
 *   BI_MODE_LAYERCAST: z = h . W^T with exact fp32 products: h split into
 *   three bf16 parts h = p0 + p1 + p2, each part's products accumulated in
 *   fp32 on the tensor cores, z = (z0 + z1) + z2.  BI_MODE_FP32: W is f32
 *   and z is an fp32 FMA chain.
 *   lse = M + ln S over the vocabulary, reduced in BI_VOCAB_CHUNK chunks
 *   (per chunk: max, sum exp(z - max), top-1 and top-2) merged in ascending
 *   chunk order; logprob = z[target] - lse (target NULL or < 0: the argmax);
 *   argmax = lowest id among equal maxima; margin = top-1 minus top-2 logit.
 * Selective FP32 recompute ("Greedy Decoding Is Not Precision-Invariant",
 *   method section: recompute the LM head in FP32 only when the top-two logit
 *   margin falls below a threshold): in BI_MODE_BF16, rows with
 *   margin < margin_threshold are recomputed from the f32 h at FP32 accuracy:
 *   h is split exactly into three bf16 parts (h = p0 + p1 + p2; 8+8+8
 *   significant bits), each product with W is exact, the three products are
 *   accumulated in fp32 on the tensor cores and added as (z0 + z1) + z2.
 *   p0 = bf16(h) is the main-pass input.  For B <= 42 one GEMM pass over W
 *   computes the main logits and the parts of every row (3B token rows in
 *   one 128-row token tile, W read once); for larger B a second pass over W
 *   computes p1.W^T and p2.W^T of the flagged rows only, when there are any.
 *   Their lse, logprob and argmax are replaced; margin keeps the bf16-path
 *   value that triggered the recompute;
 *   recomputed[b] = 1.  margin_threshold <= 0 disables it.  In LAYERCAST the
 *   main pass is already fp32 and recomputed[b] = 0.
 * Outputs (device, [B]): logprob f32, lse f32, argmax int32, margin f32,
 *   recomputed uint8; logits (optional, f32 [B][V]): the main-pass logits
 *   (bf16-path logits in BI_MODE_BF16; rows are not replaced by the recompute).
 * Requirements: H % 64 == 0, V % 64 == 0. */
size_t bi_lmhead_workspace_size(int B, int H, int V, int mode);
int bi_lmhead_logprob(const float* h, const void* W, const int32_t* target, int B, int H, int V,
                      float margin_threshold, int mode, float* logprob, float* lse, int32_t* argmax, float* margin,
                      uint8_t* recomputed, float* logits, void* ws, size_t ws_bytes, void* stream);

/* The LM head in stages, for callers that shard the vocabulary across ranks
 * (tensor parallelism: "Meituan bitwise train/infer consistency", TP item --
 * each rank computes its vocabulary rows over the full K, the logits are
 * gathered, and the fixed-order reduction runs on the whole row).
 * bi_lmhead_split: out (bf16 [parts*B][H], device) = the GEMM rows of
 *   bi_lmhead_logprob: rows 0..B-1 = bf16(h) (round to nearest even); with
 *   parts == 3 also the exact residual parts p1 (rows B..2B-1) and p2 (rows
 *   2B..3B-1), h = p0 + p1 + p2.
 * bi_lmhead_from_logits: z (f32 [parts*B][V], device) = those rows times W^T
 *   (any row-sharded GEMM whose shards are concatenated by vocabulary id);
 *   runs the vocabulary-chunk partials, the ascending merge, the margin test
 *   and -- parts == 3 and margin_threshold > 0 -- the FP32 recompute of the
 *   flagged rows from (z0 + z1) + z2, with the outputs of bi_lmhead_logprob.
 *   Given the same logits, every output is bitwise that of bi_lmhead_logprob
 *   (the same kernels, arguments and order).  Workspace:
 *   bi_lmhead_logits_workspace_size(B, V) bytes. */
int bi_lmhead_split(const float* h, int B, int H, int parts, void* out, void* stream);
size_t bi_lmhead_logits_workspace_size(int B, int V);
int bi_lmhead_from_logits(const float* z, int B, int V, int parts, const int32_t* target, float margin_threshold,
                          float* logprob, float* lse, int32_t* argmax, float* margin, uint8_t* recomputed, void* ws,
                          size_t ws_bytes, void* stream);

/* LM-head logprob for callers that cannot allocate device memory.  (No
 * counterpart on the pages: this is an interface convenience, not part of
 * the method.)  Some callers cannot call cudaMalloc -- code running while a
 * caching allocator owns all device memory, plug-ins handed only their inputs
 * and outputs, request paths where allocation is forbidden -- so this variant
 * takes no workspace: its scratch is a fixed array of BI_NOALLOC_SCRATCH_BYTES
 * inside the library, which every GPU that loads the library keeps until the
 * process exits.  Arguments and results are those of bi_lmhead_logprob, and
 * so is the arithmetic (the results are bit-identical).
 *  - Calls whose scratch need exceeds BI_NOALLOC_SCRATCH_BYTES are rejected
 *    with BI_ERR_WORKSPACE and a message; at hidden 4096 / vocab 128256 that
 *    allows up to 53 rows in BI_MODE_BF16 (bi_lmhead_workspace_size gives
 *    the need of the recompute-enabled case).
 *  - The first call on a device looks up the array's device address (once per
 *    device, with that device current); make that first call before any
 *    stream capture.  The address is kept for the life of the process: a
 *    cudaDeviceReset destroys the array with everything else on the device,
 *    so do not call this entry point again in that process after a reset.
 *  - All calls share the one array: calls whose GPU work overlaps (different
 *    streams, or host threads racing) corrupt each other's scratch.  Issue
 *    them in one stream order.  Nothing in the array needs to start zeroed.
 *  - It allocates nothing: no cudaMalloc/cudaFree, no allocating library call. */
#define BI_NOALLOC_SCRATCH_BYTES (80 << 20)
int bi_lmhead_logprob_noalloc(const float* h, const void* W, const int32_t* target, int B, int H, int V,
                              float margin_threshold, int mode, float* logprob, float* lse, int32_t* argmax,
                              float* margin, uint8_t* recomputed, float* logits, void* stream);

/* ------------------------------------------------------------ Decode step
 * A whole decoder forward for a batch of tokens (any mix of prefill chunks and
 * decode tokens of many slots: continuous batching), followed by the LM-head
 * logprob above for the tokens that ask for it.  This is the pages' unit of
 * consistency: "Meituan bitwise train/infer consistency" (opening summary and
 * key-practices list) asks that a token's probability be bit-identical
 * whichever way it is computed -- Prefill or Decode, any batch -- and every
 * step here is one of the fixed-order calls above, so a token's logprob
 * depends only on its own sequence.  Weights: bf16, caller-owned, device
 * pointers; layouts below.  Architecture (the pages are silent; the
 * workloads' Llama-3.1-8B and Qwen2.5-7B shapes): pre-norm decoder with
 * RMSNorm, GQA attention with rotate-half RoPE, SwiGLU MLP, untied LM head,
 * no biases. */
typedef struct {
  int n_layers, hidden, n_heads, n_kv_heads, head_dim, ffn, vocab;
  float eps;
  int mode;    /* BI_MODE_BF16 or BI_MODE_LAYERCAST */
  int variant; /* BI_VARIANT_INVARIANT or BI_VARIANT_FAST */
  float margin_threshold;
} bi_model_desc;

typedef struct {
  const void* embed;      /* bf16 [V][H] */
  const void* lm_head;    /* bf16 [V][H] */
  const void* final_norm; /* bf16 [H] */
  const void* attn_norm;  /* bf16 [L][H] */
  const void* ffn_norm;   /* bf16 [L][H] */
  const void* w_qkv;      /* bf16 [L][(Hq + 2 Hkv) d][H]: q rows, k rows, v rows; each q and k head in
                             the PAIRED row order: in every 32-row block b of a head, rows 0..15 are
                             elements 16b..16b+15 and rows 16..31 their rotate-half partners
                             d/2+16b..d/2+16b+15 (so RoPE can run in the projection's epilogue);
                             v heads in natural order */
  const void* w_o;        /* bf16 [L][H][Hq d] */
  const void* w_gu;       /* bf16 [L][2F][H], gate/up interleaved by BI_GU_INTERLEAVE */
  const void* w_down;     /* bf16 [L][H][F] */
  const float* rope;      /* f32 table from bi_rope_table_fill */
  int rope_max_pos;
} bi_weights;

/* A context only records the model description and the caller's weight and
 * KV-cache pointers (no device memory, no launch); it checks that the shapes
 * are ones the kernels implement (the pages are silent on interfaces). */
typedef struct bi_ctx bi_ctx;
int bi_ctx_create(const bi_model_desc* desc, const bi_weights* w, const bi_kv_layout* kv, bi_ctx** out);
int bi_ctx_destroy(bi_ctx* ctx);

typedef struct {
  int n_tokens;
  const int32_t* ids;       /* device [n_tokens] token ids */
  const int32_t* slot;      /* device [n_tokens] KV slot of each token */
  const int32_t* pos;       /* device [n_tokens] position of each token in its slot */
  const int32_t* slot_host; /* host copies of slot and pos (validation, planning) */
  const int32_t* pos_host;
  const int32_t* lm_row;    /* device [n_tokens]: output row of the token, or -1 */
  int n_lm;                 /* number of output rows (tokens with lm_row >= 0) */
  const int32_t* target;    /* device [n_lm]: token whose logprob is wanted; NULL or -1 = greedy */
} bi_batch;

typedef struct {
  float* logprob;      /* device [n_lm] */
  float* lse;          /* device [n_lm] */
  int32_t* argmax;     /* device [n_lm]  (greedy next token) */
  float* margin;       /* device [n_lm] */
  uint8_t* recomputed; /* device [n_lm] */
  float* logits;       /* optional device [n_lm][V] */
  float* h;            /* optional device [n_lm][H]: final norm output, f32 */
} bi_step_out;

size_t bi_decode_workspace_size(const bi_ctx* ctx, int max_tokens, int max_lm_rows, int max_pos);
int bi_decode_step(bi_ctx* ctx, const bi_batch* batch, const bi_step_out* out, void* ws, size_t ws_bytes,
                   void* stream);

/* Embedding gather (the first step of bi_decode_step, for callers that run
 * the layers themselves, e.g. a tensor-parallel orchestration): x[t] =
 * embed[ids[t]] in the activation dtype of mode (bf16 values, exact in f32).
 * ids: device int32 [T]; embed: bf16 [V][H]; x: [T][H].  An id outside
 * [0, V) sets the index bit of the device error word and gives a zero row. */
int bi_embed(const int32_t* ids, const void* embed, int T, int H, int V, int mode, void* x, void* stream);

/* Greedy feedback for a device-resident decode loop: for b < B,
 * ids[b] = argmax[b] and pos[b] += 1 (device int32 arrays). */
int bi_greedy_advance(const int32_t* argmax, int32_t* ids, int32_t* pos, int B, void* stream);

/* ----------------------------------------------------------- Synthetic init
 * Device twin of the seeded generator used for the synthetic workloads:
 * SplitMix64 counters -> Irwin-Hall(12) normal -> bf16(f32(z * std)).
 * Writes logical element i (row i / cols, column i % cols) of a [rows][cols]
 * tensor of stream `key`, starting at logical element 0, to
 *   dst[dst_row(i / cols) * cols + i % cols], where
 *   dst_row(r) = r                                   if interleave == 0,
 *   dst_row(r) = (r / g) * 2g + phase * g + r % g    if interleave == g > 0
 * (phase 0 = gate rows, 1 = up rows of a BI_GU_INTERLEAVE fused weight),
 *   dst_row(r) = (r / d) * d + paired(r % d)         if interleave == -d
 * (d = 64 or 128: the paired row order of q/k heads in bi_weights.w_qkv).
 * Not part of the method: it only produces inputs without a host round trip. */
int bi_synth_fill_bf16(uint16_t* dst, int64_t rows, int64_t cols, uint64_t key, double std, int interleave,
                       int phase, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* BI_H */
