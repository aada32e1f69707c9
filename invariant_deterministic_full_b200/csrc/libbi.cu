// libbi: batch-invariant decoder forward + LM-head logprob for sm_100a.
// One translation unit: the kernels live in the included .cuh files; this
// file holds the C ABI declared in include/bi.h (argument checks, workspace
// carving, launches) and the decode-step orchestration.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <vector>

#include <nvtx3/nvToolsExt.h>  // header-only NVTX v3: ranges cost a pointer check unless a profiler attaches

#include "host_common.cuh"
#include "gemm.cuh"
#include "norm_rope.cuh"
#include "attention.cuh"
#include "lmhead.cuh"
#include "synth_fill.cuh"

namespace bi {

// Workspace carving: 256-byte aligned sub-buffers.  With base == nullptr it
// only measures.
struct Carver {
  uint8_t* base;
  size_t used = 0;
  explicit Carver(void* b) : base(reinterpret_cast<uint8_t*>(b)) {}
  template <typename T>
  T* take(size_t count) {
    used = (used + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + used) : nullptr;
    used += count * sizeof(T);
    return p;
  }
};

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
static bool mode_ok(int mode) { return mode == BI_MODE_BF16 || mode == BI_MODE_LAYERCAST || mode == BI_MODE_FP32; }
// Activations and the KV cache are f32 in LayerCast and FP32 modes.
static int act_f32(int mode) { return mode != BI_MODE_BF16 ? 1 : 0; }

// ------------------------------------------------------------------ GEMM
static int gemm_run(const void* x, int ldx, const void* w, void* y, int ldy, int y_dtype, int M, int N, int K, int epi,
                    const bi_epi_args* ea, int mode, int variant, void* ws, size_t ws_bytes, cudaStream_t st,
                    int n_full = 0) {
  const bool rope = epi == BI_EPI_ROPE_KV_APPEND;
  BI_REQUIRE(w && ((x && (y || rope)) || M == 0), BI_ERR_INVALID_ARG, "bi_gemm: NULL pointer");
  BI_REQUIRE(M >= 0 && N > 0 && K > 0, BI_ERR_INVALID_ARG, "bi_gemm: bad sizes M=%d N=%d K=%d", M, N, K);
  BI_REQUIRE(n_full == 0 || (n_full >= N && n_full % 64 == 0), BI_ERR_INVALID_ARG,
             "bi_gemm: n_full=%d must be 0 or the full matrix's rows (>= N=%d, a multiple of 64)", n_full, N);
  BI_REQUIRE(K % 64 == 0 && N % 64 == 0, BI_ERR_UNSUPPORTED, "bi_gemm: need K %% 64 == 0 and N %% 64 == 0 (N=%d K=%d)",
             N, K);
  BI_REQUIRE(ldx >= K && ldx % 8 == 0, BI_ERR_UNSUPPORTED, "bi_gemm: ldx=%d must be >= K and a multiple of 8", ldx);
  BI_REQUIRE(epi == BI_EPI_NONE || epi == BI_EPI_SWIGLU || rope, BI_ERR_INVALID_ARG, "bi_gemm: bad epilogue %d", epi);
  const int n_out = epi == BI_EPI_SWIGLU ? N / 2 : N;
  BI_REQUIRE(rope || ldy >= n_out, BI_ERR_INVALID_ARG, "bi_gemm: ldy=%d < output columns %d", ldy, n_out);
  BI_REQUIRE(aligned16(x) && aligned16(w), BI_ERR_UNSUPPORTED, "bi_gemm: x and w must be 16-byte aligned");
  BI_REQUIRE(mode_ok(mode), BI_ERR_INVALID_ARG, "bi_gemm: bad mode %d", mode);
  BI_REQUIRE(y_dtype == BI_DTYPE_BF16 || y_dtype == BI_DTYPE_F32, BI_ERR_INVALID_ARG, "bi_gemm: bad y dtype");
  BI_REQUIRE(rope == (ea != nullptr), BI_ERR_INVALID_ARG, "bi_gemm: epilogue arguments %s",
             rope ? "missing for BI_EPI_ROPE_KV_APPEND" : "given for an epilogue that takes none");
  RopeEpi re{};
  if (rope) {
    BI_REQUIRE(mode == BI_MODE_BF16 && variant == BI_VARIANT_INVARIANT, BI_ERR_UNSUPPORTED,
               "bi_gemm: BI_EPI_ROPE_KV_APPEND needs BI_MODE_BF16 and the invariant variant");
    const bi_kv_layout* kv = ea->kv;
    BI_REQUIRE(kv && kv->k && kv->v && ea->rope && ea->q_out && ea->slot && ea->pos, BI_ERR_INVALID_ARG,
               "bi_gemm: NULL RoPE/KV epilogue argument");
    BI_REQUIRE(kv->dtype == BI_DTYPE_BF16, BI_ERR_INVALID_ARG, "bi_gemm: the RoPE/KV epilogue needs a bf16 cache");
    BI_REQUIRE(kv->head_dim == 64 || kv->head_dim == 128, BI_ERR_UNSUPPORTED, "bi_gemm: head_dim %d", kv->head_dim);
    BI_REQUIRE(ea->n_heads > 0 && kv->n_kv_heads > 0 && ea->n_heads % kv->n_kv_heads == 0, BI_ERR_INVALID_ARG,
               "bi_gemm: Hq=%d Hkv=%d", ea->n_heads, kv->n_kv_heads);
    BI_REQUIRE(N == (ea->n_heads + 2 * kv->n_kv_heads) * kv->head_dim, BI_ERR_INVALID_ARG,
               "bi_gemm: N=%d is not (Hq + 2 Hkv) * head_dim", N);
    BI_REQUIRE(ea->layer >= 0 && ea->layer < kv->n_layers && kv->n_slots > 0 && kv->capacity > 0 &&
                   ea->rope_max_pos > 0,
               BI_ERR_INVALID_ARG, "bi_gemm: bad cache layer/shape");
    BI_REQUIRE(aligned16(ea->q_out) && aligned16(kv->k) && aligned16(kv->v), BI_ERR_UNSUPPORTED,
               "bi_gemm: q_out and the cache must be 16-byte aligned");
    re = RopeEpi{ea->rope, ea->rope_max_pos, ea->q_out, kv->k, kv->v, ea->slot, ea->pos,
                 ea->n_heads, kv->n_kv_heads, kv->head_dim, ea->layer, kv->n_layers, kv->n_slots, kv->capacity};
  }
  if (M == 0) return BI_OK;
  const int y_f32 = y_dtype == BI_DTYPE_F32;
  if (mode == BI_MODE_FP32)
    return gemm_f32(reinterpret_cast<const float*>(x), ldx, w, y, ldy, y_f32, M, N, K, epi, nullptr, st, true);
  if (mode == BI_MODE_LAYERCAST)
    return gemm_layercast(reinterpret_cast<const float*>(x), ldx, w, y, ldy, y_f32, M, N, K, epi, ws, ws_bytes, st,
                          n_full);
  return gemm_bf16(x, ldx, w, y, ldy, y_f32, M, N, K, epi, variant, ws, ws_bytes, st, nullptr, 1,
                   rope ? &re : nullptr, n_full);
}

// ------------------------------------------------------------------ attention
static int attn_chunk_for(int T, int variant) {
  if (variant != BI_VARIANT_FAST) return ATT_CHUNK;
  // FAST: KV split chosen from the batch size (more, smaller chunks for small batches).
  return T <= 4 ? 64 : (T <= 16 ? 128 : 256);
}

// Tokens per attention launch: as many as fit a 640 MB partials workspace (at
// least ATT_TOKEN_GROUP), so a long prefill is one or a few large launches.
constexpr size_t ATT_PART_BUDGET = size_t(640) << 20;
static int attn_token_group(int T, int Hq, int d, int max_chunks) {
  const size_t per_tok = (size_t)Hq * max_chunks * (d + 4) * sizeof(float);
  const size_t by_budget = ATT_PART_BUDGET / per_tok;
  return (int)std::min<size_t>((size_t)T, std::max<size_t>(ATT_TOKEN_GROUP, std::min<size_t>(by_budget, 1u << 20)));
}
static size_t attn_ws_bytes(int T, int Hq, int d, int max_pos, int chunk) {
  const int max_chunks = max_pos / chunk + 1;
  const int tg = attn_token_group(T, Hq, d, max_chunks);
  return (size_t)tg * Hq * max_chunks * (d + 4) * sizeof(float) + 256;
}

static int attn_set_smem_attrs() {
  static bool done = false;
  if (done) return BI_OK;
  BI_CHECK_CUDA(cudaFuncSetAttribute(attn_partial_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)att_smem_bytes(4, 128, 1)));
  BI_CHECK_CUDA(cudaFuncSetAttribute(attn_partial_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)att_smem_bytes(8, 128, 1)));
  BI_CHECK_CUDA(cudaFuncSetAttribute(attn_partial_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)att_smem_bytes(16, 128, 1)));
  BI_CHECK_CUDA(cudaFuncSetAttribute(attn_partial_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)att_smem_bytes(32, 128, 1)));
  BI_CHECK_CUDA(cudaFuncSetAttribute(attn_tc_kernel<2, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)atc_smem_bytes(2, 4)));
  BI_CHECK_CUDA(cudaFuncSetAttribute(attn_tc_kernel<4, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)atc_smem_bytes(4, 2)));
  BI_CHECK_CUDA(cudaFuncSetAttribute(attn_pre_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)atp_smem_bytes()));
  BI_CHECK_CUDA(cudaFuncSetAttribute(attn_dec_kernel<4, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)atd_smem_bytes(4, 4)));
  BI_CHECK_CUDA(cudaFuncSetAttribute(attn_dec_kernel<3, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)atd_smem_bytes(3, 8)));
  done = true;
  return BI_OK;
}

// np: pairs per group of the CUDA-core kernel (LayerCast, or head_dim 64); the
// bf16 head_dim-128 path runs on tensor cores with 16-row pair tiles.
//
// Tensor-core kernel: a CTA walks a segment of consecutive chunks of one
// (block, kv head).  With enough (block, kv head) units (at least two thirds
// of the SM count), one segment spans all chunks and the CTA also merges (no
// merge launch);
// otherwise the chunks are cut into segments so that about two CTAs per SM
// run, and the merge kernel combines the partials.  Either way the chunk
// partials and the merge are the same computations (work assignment only).
// *merged reports whether this launch wrote the final outputs itself.
static int attn_launch(int np, const CUtensorMap& tk, const CUtensorMap& tv, const AttnPlan& plan, AttnArgs a,
                       cudaStream_t st, bool* merged) {
  *merged = false;
  if (!a.f32 && a.d == 128) {
    const bool single = np <= 16;  // decode blocks: one token, G pairs
    const bool dec = single && a.G <= 8;  // the decode schedule: one 8-pair tile, at most ATD_SEG chunks per CTA
    const int units = plan.n * a.Hkv;
    const int target = 2 * num_sms();
    int n_seg = units >= target / 3 ? 1 : std::min(a.max_chunks, (target + units - 1) / units);
    a.seg_len = (a.max_chunks + n_seg - 1) / n_seg;
    if (dec) a.seg_len = std::min(a.seg_len, ATD_SEG);
    n_seg = (a.max_chunks + a.seg_len - 1) / a.seg_len;
    a.merge_in_cta = n_seg == 1;
    *merged = a.merge_in_cta != 0;
    const dim3 grid(plan.n, n_seg, a.Hkv);
    // decode: 4-pair rows for kv heads of at most 4 q heads (a 4-deep ring), else
    // 8 (3-deep); either way two CTAs fit an SM
    if (dec && a.G <= 4)
      BI_TRY(launch(attn_dec_kernel<4, 4>, grid, dim3(ATC_THREADS), atd_smem_bytes(4, 4), st, tk, tv, plan, a));
    else if (dec)
      BI_TRY(launch(attn_dec_kernel<3, 8>, grid, dim3(ATC_THREADS), atd_smem_bytes(3, 8), st, tk, tv, plan, a));
    else if (single && a.G <= 16)
      BI_TRY(launch(attn_tc_kernel<2, 4>, grid, dim3(ATC_THREADS), atc_smem_bytes(2, 4), st, tk, tv, plan, a));
    else  // prefill blocks: the chunk's K and V rows resident for all pair groups
      BI_TRY(launch(attn_pre_kernel, grid, dim3(ATP_THREADS), atp_smem_bytes(), st, tk, tv, plan, a));
    return BI_OK;
  }
  a.seg_len = 1;
  a.merge_in_cta = 0;
  const dim3 grid(plan.n, a.max_chunks, a.Hkv);
  const size_t smem = att_smem_bytes(np, a.d, a.f32);
  switch (np) {
    case 4: BI_TRY(launch(attn_partial_kernel<4>, dim3(grid), dim3(ATT_THREADS), smem, st, tk, tv, plan, a)); break;
    case 8: BI_TRY(launch(attn_partial_kernel<8>, dim3(grid), dim3(ATT_THREADS), smem, st, tk, tv, plan, a)); break;
    case 16: BI_TRY(launch(attn_partial_kernel<16>, dim3(grid), dim3(ATT_THREADS), smem, st, tk, tv, plan, a)); break;
    default: BI_TRY(launch(attn_partial_kernel<32>, dim3(grid), dim3(ATT_THREADS), smem, st, tk, tv, plan, a)); break;
  }
  return BI_OK;
}

// early_kv: the caller guarantees that slot, pos and the cache rows below the
// step's positions were written before the kernel preceding this launch (the
// decode step); with one token per slot the decode kernel may then read them
// before its dependency wait.
static int attention_run(const void* q, const bi_kv_layout* kv, int layer, const int32_t* slot, const int32_t* pos,
                         const int32_t* slot_h, const int32_t* pos_h, void* out, int T, int Hq, float scale, int mode,
                         int variant, void* ws, size_t ws_bytes, cudaStream_t st, bool early_kv = false) {
  BI_REQUIRE(q && kv && slot && pos && slot_h && pos_h && out, BI_ERR_INVALID_ARG, "bi_attention: NULL pointer");
  BI_REQUIRE(kv->k && kv->v, BI_ERR_INVALID_ARG, "bi_attention: NULL KV cache");
  const int d = kv->head_dim, Hkv = kv->n_kv_heads;
  BI_REQUIRE(d == 64 || d == 128, BI_ERR_UNSUPPORTED, "bi_attention: head_dim %d (need 64 or 128)", d);
  BI_REQUIRE(Hkv > 0 && Hq > 0 && Hq % Hkv == 0, BI_ERR_INVALID_ARG, "bi_attention: Hq=%d Hkv=%d", Hq, Hkv);
  BI_REQUIRE(layer >= 0 && layer < kv->n_layers, BI_ERR_INVALID_ARG, "bi_attention: layer %d", layer);
  BI_REQUIRE(mode_ok(mode), BI_ERR_INVALID_ARG, "bi_attention: bad mode %d", mode);
  const int f32 = act_f32(mode);
  BI_REQUIRE(kv->dtype == (f32 ? BI_DTYPE_F32 : BI_DTYPE_BF16), BI_ERR_INVALID_ARG,
             "bi_attention: KV dtype does not match the mode");
  if (T == 0) return BI_OK;
  const int G = Hq / Hkv;
  BI_REQUIRE(G <= ATT_MAX_PAIRS, BI_ERR_UNSUPPORTED, "bi_attention: %d q heads per kv head (max %d)", G, ATT_MAX_PAIRS);
  const int chunk = attn_chunk_for(T, variant);
  // query-block size (work assignment only): a CTA streams one KV chunk and loops over
  // the block's (query, head) pairs 32 at a time; blocks hold up to 256 pairs.
  const int QB = std::max(1, std::min(ATT_MAX_QB, 256 / G));

  // validation + plan: blocks of <= QB adjacent tokens of one slot at consecutive positions
  int max_pos = 0;
  std::vector<int2> blocks;
  blocks.reserve(T);
  for (int t = 0; t < T; ++t) {
    const int s = slot_h[t], p = pos_h[t];
    BI_REQUIRE(s >= 0 && s < kv->n_slots, BI_ERR_INVALID_ARG, "bi_attention: token %d slot %d out of range", t, s);
    BI_REQUIRE(p >= 0 && p < kv->capacity, BI_ERR_CAPACITY, "bi_attention: token %d position %d >= capacity %d", t, p,
               kv->capacity);
    max_pos = std::max(max_pos, p);
    const bool extend = !blocks.empty() && slot_h[t - 1] == s && pos_h[t - 1] + 1 == p &&
                        blocks.back().y < QB && (t - blocks.back().x) == blocks.back().y;
    if (extend)
      blocks.back().y++;
    else
      blocks.push_back(make_int2(t, 1));
  }
  bool one_per_slot = early_kv;
  if (one_per_slot) {
    std::vector<char> seen(kv->n_slots, 0);
    for (int t = 0; t < T && one_per_slot; ++t) {
      one_per_slot = !seen[slot_h[t]];
      seen[slot_h[t]] = 1;
    }
  }
  const int max_chunks = max_pos / chunk + 1;
  const size_t need = attn_ws_bytes(T, Hq, d, max_pos, chunk);
  const int tg = attn_token_group(T, Hq, d, max_chunks);
  BI_REQUIRE(ws && ws_bytes >= need, BI_ERR_WORKSPACE, "bi_attention: workspace %zu < %zu", ws_bytes, need);

  const int esz = f32 ? 4 : 2;
  const uint64_t rows = (uint64_t)kv->n_slots * kv->n_layers * Hkv * kv->capacity;
  CUtensorMap tk, tv;
  const CUtensorMapDataType dt = f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  // 3-D views {128-byte piece of a row, row, piece}: a 64-row box of all pieces is
  // one TMA operation landing as [piece][64 rows][128 B] swizzled slabs.
  const uint32_t ninner = (uint32_t)(d * esz / 128);
  const uint64_t kdims[3] = {(uint64_t)(128 / esz), rows, ninner};
  const uint64_t kstr[2] = {(uint64_t)d * esz, 128};
  const uint32_t kbox[3] = {(uint32_t)(128 / esz), 64, ninner};
  BI_TRY(encode_tmap_3d(&tk, dt, kv->k, kdims, kstr, kbox, CU_TENSOR_MAP_SWIZZLE_128B));
  BI_TRY(encode_tmap_3d(&tv, dt, kv->v, kdims, kstr, kbox, CU_TENSOR_MAP_SWIZZLE_128B));

  BI_TRY(attn_set_smem_attrs());
  float* part = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
  // pairs per group for single-token (decode) blocks: G rounded up to a power of two
  int np1 = 4;
  while (np1 < G) np1 *= 2;

  // Token groups of at most tg tokens bound the partials
  // workspace; a group is made of whole blocks.  Within a group, single-token
  // blocks and multi-token blocks go to two launches with different pair-group
  // sizes (work assignment only).
  size_t bi0 = 0;
  while (bi0 < blocks.size()) {
    const int t_base = blocks[bi0].x;
    size_t bi1 = bi0;
    AttnPlan p1, pm;
    p1.n = 0;
    pm.n = 0;
    while (bi1 < blocks.size() && p1.n < ATT_MAX_BLOCKS && pm.n < ATT_MAX_BLOCKS &&
           blocks[bi1].x + blocks[bi1].y - t_base <= tg) {
      if (blocks[bi1].y == 1)
        p1.blk[p1.n++] = blocks[bi1++];
      else
        pm.blk[pm.n++] = blocks[bi1++];
    }
    if (bi1 == bi0) return set_error(BI_ERR_UNSUPPORTED, "bi_attention: planning failed");
    const int t_end = blocks[bi1 - 1].x + blocks[bi1 - 1].y;
    AttnArgs a;
    a.q = q; a.slot = slot; a.pos = pos; a.part = part; a.t_base = t_base;
    a.Hq = Hq; a.Hkv = Hkv; a.G = G; a.d = d; a.chunk = chunk; a.max_chunks = max_chunks;
    a.layer = layer; a.n_layers = kv->n_layers; a.cap = kv->capacity; a.f32 = f32; a.scale = scale;
    a.pre_kv = one_per_slot ? 1 : 0;
    a.out = out;
    bool m1 = true, mm = true;
    if (p1.n) BI_TRY(attn_launch(np1, tk, tv, p1, a, st, &m1));
    if (pm.n) BI_TRY(attn_launch(ATT_MAX_PAIRS, tk, tv, pm, a, st, &mm));
    if (!(m1 && mm)) {  // merges every token of the group (rewriting merged ones with the same bits)
      const int nw = (t_end - t_base) * Hq;
      BI_TRY(launch(attn_merge_kernel, dim3((nw * 32 + 255) / 256), dim3(256), 0, st, part, pos, out, t_base,
                    t_end - t_base, Hq, d, chunk, max_chunks, f32));
    }
    bi0 = bi1;
  }
  return BI_OK;
}

// ------------------------------------------------------------------ LM head
// LM-head recompute layouts.  One pass (B <= LM_ONE_PASS_ROWS): the GEMM runs
// over 3B rows -- bf16(h) then the two exact residual parts of every row --
// which fit one 128-row token tile of the tensor-core MMA, so W is read once
// and the flagged rows' FP32 logits come for free (the MMA costs the same for
// 3 or 126 live rows).  Two passes (larger B): the main GEMM over B
// rows, then one more pass over W for the two residual parts of the flagged
// rows only (none when no row is flagged); the part bf16(h) is the main
// pass's.  Both compute every logit with the same per-row arithmetic.
constexpr int LM_ONE_PASS_ROWS = 42;
struct LmWs {
  uint16_t* hs;     // bf16 GEMM input: [B][H], or [3B][H] in the one-pass layout
  float* logits;    // [B or 3B][V] (LayerCast: [B][V] unless the caller's buffer is used)
  LmPart* part;
  uint8_t* flag;
  int32_t* list;
  int* count;
  uint16_t* hc2;    // two-pass: [2B][H] residual parts p1, p2 of the flagged rows
  float* logits_c;  // two-pass: [2B][V] their logits
  void* lc;         // LayerCast: the tensor-core GEMM's split rows and partial products
  size_t lc_bytes;
};
// LayerCast LM head: vocabulary columns per tensor-core pass (bounds its workspace)
constexpr int LM_LC_COLS = 16384;
// parts: 3 in bf16 mode with the recompute enabled, else 1
static LmWs lm_carve(Carver& cv, int B, int H, int V, int mode, bool own_logits, int parts) {
  const int nch = (V + LM_CHUNK - 1) / LM_CHUNK;
  LmWs w{};
  const bool bf = mode == BI_MODE_BF16;
  const int rows = (bf && parts == 3 && B <= LM_ONE_PASS_ROWS) ? 3 * B : B;
  w.hs = bf ? cv.take<uint16_t>((size_t)rows * H) : nullptr;
  w.logits = (bf || own_logits) ? cv.take<float>((size_t)(bf ? rows : B) * V) : nullptr;
  w.part = cv.take<LmPart>((size_t)(rows == 3 * B ? 2 : 1) * B * nch);  // one pass: main and exact partials
  w.flag = cv.take<uint8_t>(B);
  w.list = cv.take<int32_t>(B);
  w.count = cv.take<int>(1);
  if (bf && parts == 3 && B > LM_ONE_PASS_ROWS) {
    w.hc2 = cv.take<uint16_t>((size_t)2 * B * H);
    w.logits_c = cv.take<float>((size_t)2 * B * V);
  }
  if (mode == BI_MODE_LAYERCAST) {
    w.lc_bytes = lc_ws_bytes(B, V, H, LM_LC_COLS);
    w.lc = cv.take<uint8_t>(w.lc_bytes);
  }
  return w;
}
static int lm_parts(int mode, float thresh) { return mode == BI_MODE_BF16 && thresh > 0.f ? 3 : 1; }

static int lmhead_run(const float* h, const void* W, const int32_t* target, int B, int H, int V, float thresh, int mode,
                      float* logprob, float* lse, int32_t* argmax, float* margin, uint8_t* recomputed, float* logits,
                      void* ws, size_t ws_bytes, cudaStream_t st) {
  BI_REQUIRE(h && W && logprob && lse && argmax && margin && recomputed, BI_ERR_INVALID_ARG,
             "bi_lmhead_logprob: NULL pointer");
  BI_REQUIRE(B >= 0 && H > 0 && V > 0, BI_ERR_INVALID_ARG, "bi_lmhead_logprob: bad sizes");
  BI_REQUIRE(H % 64 == 0 && V % 64 == 0, BI_ERR_UNSUPPORTED, "bi_lmhead_logprob: need H, V multiples of 64");
  BI_REQUIRE(mode_ok(mode), BI_ERR_INVALID_ARG, "bi_lmhead_logprob: bad mode");
  BI_REQUIRE(aligned16(h) && aligned16(W), BI_ERR_UNSUPPORTED, "bi_lmhead_logprob: h and W must be 16-byte aligned");
  if (B == 0) return BI_OK;
  const int parts = lm_parts(mode, thresh);
  Carver probe(nullptr);
  lm_carve(probe, B, H, V, mode, logits == nullptr, parts);
  BI_REQUIRE(ws && ws_bytes >= probe.used + 256, BI_ERR_WORKSPACE, "bi_lmhead_logprob: workspace %zu < %zu", ws_bytes,
             probe.used + 256);
  Carver cv(reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255)));
  LmWs w = lm_carve(cv, B, H, V, mode, logits == nullptr, parts);
  const int nch = (V + LM_CHUNK - 1) / LM_CHUNK;
  const bool one_pass = parts == 3 && B <= LM_ONE_PASS_ROWS;
  float* z;
  if (mode == BI_MODE_BF16) {
    // One pass over W: rows 0..B-1 of the GEMM input are bf16(h) (the main
    // pass); with the recompute enabled, rows B..3B-1 hold the exact split
    // parts, whose logits are combined ((z0 + z1) + z2) only for flagged rows.
    const size_t n = (size_t)B * H;
    const int sp = one_pass ? 3 : 1;
    z = w.logits;
    BI_TRY(launch(lm_split_kernel, dim3((int)std::min<size_t>((n + 255) / 256, 4096)), dim3(256), 0, st, h, w.hs, n,
                  sp));
    BI_TRY(gemm_bf16(w.hs, H, W, z, V, 1, sp * B, V, H, BI_EPI_NONE, BI_VARIANT_INVARIANT, nullptr, 0, st));
    if (logits)
      BI_CHECK_CUDA(cudaMemcpyAsync(logits, z, (size_t)B * V * sizeof(float), cudaMemcpyDeviceToDevice, st));
  } else if (mode == BI_MODE_LAYERCAST) {
    // exact products of fp32 h with the bf16 W on the tensor cores (three bf16
    // parts of h, fp32 accumulation), as the LayerCast projections
    z = logits ? logits : w.logits;
    BI_TRY(gemm_layercast(h, H, W, z, V, 1, B, V, H, BI_EPI_NONE, w.lc, w.lc_bytes, st, V, LM_LC_COLS));
  } else {
    z = logits ? logits : w.logits;
    BI_TRY(gemm_f32(h, H, W, z, V, 1, B, V, H, BI_EPI_NONE, nullptr, st, true));
  }
  // FP32 logits of the flagged rows: h = p0 + p1 + p2 exactly (bf16 parts), so
  // h.W^T = ((p0.W^T + p1.W^T) + p2.W^T) with exact products and fp32
  // accumulation on the tensor cores.  One pass: the GEMM above computed them
  // for every row, and one partials launch and one merge launch serve both
  // paths (the merge picks the exact one for the flagged rows).  Two passes:
  // the main path first, then one more pass over W for the flagged rows only
  // (row count read on the device).
  const bool fused = parts == 3 && one_pass;
  const float th = mode == BI_MODE_BF16 ? thresh : 0.f;
  BI_TRY(launch(lm_partial_kernel, dim3((nch + LM_CPB - 1) / LM_CPB, fused ? 2 * B : B), dim3(32 * LM_CPB), 0, st, z,
                (size_t)V, V, target, nullptr, nullptr, w.part, nch, fused ? 4 : 1, fused ? B : 0, nullptr));
  BI_TRY(launch(lm_merge_kernel, dim3((B * 32 + 127) / 128), dim3(128), 0, st, w.part, nch, B, nullptr, nullptr, target,
                th, fused ? 2 : 0, logprob, lse, argmax, margin, recomputed, w.flag));
  if (parts == 3 && !one_pass) {
    BI_TRY(launch(lm_compact_kernel, dim3(B), dim3(256), 0, st, w.flag, B, h, H, w.list, w.count, w.hc2));
    BI_TRY(gemm_bf16(w.hc2, H, W, w.logits_c, V, 1, 2 * B, V, H, BI_EPI_NONE, BI_VARIANT_INVARIANT, nullptr, 0, st,
                     w.count, 2));
    BI_TRY(launch(lm_partial_kernel, dim3((nch + LM_CPB - 1) / LM_CPB, B), dim3(32 * LM_CPB), 0, st, z, (size_t)V, V,
                  target, w.list, w.count, w.part, nch, 3, 0, w.logits_c));
    BI_TRY(launch(lm_merge_kernel, dim3((B * 32 + 127) / 128), dim3(128), 0, st, w.part, nch, B, w.count, w.list,
                  target, th, 1, logprob, lse, argmax, margin, recomputed, nullptr));
  }
  return BI_OK;
}

// The LM head's stages for callers that shard the vocabulary across ranks
// (tensor parallelism): the split of h into the GEMM rows, then everything
// after the GEMM on given logits.  The same kernels with the same arguments as
// the one-pass route of lmhead_run, so a row's results are the same bits.
struct LmStageWs {
  LmPart* part;
  uint8_t* flag;
  int32_t* list;
  int* count;
};
static LmStageWs lm_stage_carve(Carver& cv, int B, int V) {
  const int nch = (V + LM_CHUNK - 1) / LM_CHUNK;
  LmStageWs w{};
  w.part = cv.take<LmPart>((size_t)2 * B * nch);  // main and exact partials of every row
  w.flag = cv.take<uint8_t>(B);
  w.list = cv.take<int32_t>(B);
  w.count = cv.take<int>(1);
  return w;
}

static int lm_from_logits_run(const float* z, int B, int V, int parts, const int32_t* target, float thresh,
                              float* logprob, float* lse, int32_t* argmax, float* margin, uint8_t* recomputed,
                              void* ws, size_t ws_bytes, cudaStream_t st) {
  BI_REQUIRE(z && logprob && lse && argmax && margin && recomputed, BI_ERR_INVALID_ARG,
             "bi_lmhead_from_logits: NULL pointer");
  BI_REQUIRE(B >= 0 && V > 0 && (parts == 1 || parts == 3), BI_ERR_INVALID_ARG, "bi_lmhead_from_logits: bad sizes");
  if (B == 0) return BI_OK;
  Carver probe(nullptr);
  lm_stage_carve(probe, B, V);
  BI_REQUIRE(ws && ws_bytes >= probe.used + 256, BI_ERR_WORKSPACE, "bi_lmhead_from_logits: workspace %zu < %zu",
             ws_bytes, probe.used + 256);
  Carver cv(reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255)));
  LmStageWs w = lm_stage_carve(cv, B, V);
  const int nch = (V + LM_CHUNK - 1) / LM_CHUNK;
  const float th = parts == 3 ? thresh : 0.f;
  const bool fused = parts == 3 && thresh > 0.f;  // the one-pass layout's two paths in one launch each
  BI_TRY(launch(lm_partial_kernel, dim3((nch + LM_CPB - 1) / LM_CPB, fused ? 2 * B : B), dim3(32 * LM_CPB), 0, st, z,
                (size_t)V, V, target, nullptr, nullptr, w.part, nch, fused ? 4 : 1, fused ? B : 0, nullptr));
  BI_TRY(launch(lm_merge_kernel, dim3((B * 32 + 127) / 128), dim3(128), 0, st, w.part, nch, B, nullptr, nullptr,
                target, th, fused ? 2 : 0, logprob, lse, argmax, margin, recomputed, w.flag));
  return BI_OK;
}

// Failure-path check of the bounded waits: one thread waits on an mbarrier that
// nothing arrives at (no copy is in flight), so the wait runs out after kWaitNs,
// records the timeout bit and SITE_SELFTEST in the device error word and the
// kernel returns normally.
__global__ void wait_selftest_kernel() {
  pdl_wait();
  pdl_trigger();
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0u, SITE_SELFTEST);
}

}  // namespace bi

// ====================================================================== C ABI
using namespace bi;

// One NVTX range per C-ABI call, named after the call (nested calls nest).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};
#define BI_RANGE(name) const NvtxRange bi_nvtx_range_(name)

struct bi_ctx {
  bi_model_desc desc;
  bi_weights w;
  bi_kv_layout kv;
};

extern "C" {

const char* bi_last_error(void) { return t_last_error.c_str(); }
int bi_version(void) { return 1; }
long long bi_launch_count(void) { return g_launches; }
int bi_num_sms(int device) {
  int n = -1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) return -1;
  return n;
}

int bi_device_error(unsigned* flags, int reset) {
  unsigned v = 0, site = 0;
  BI_CHECK_CUDA(cudaMemcpyFromSymbol(&v, g_dev_error, sizeof(v)));
  BI_CHECK_CUDA(cudaMemcpyFromSymbol(&site, g_dev_site, sizeof(site)));
  if (flags) *flags = (v & 0xffu) | (site << 8);
  if (reset) {
    unsigned z = 0;
    BI_CHECK_CUDA(cudaMemcpyToSymbol(g_dev_error, &z, sizeof(z)));
    BI_CHECK_CUDA(cudaMemcpyToSymbol(g_dev_site, &z, sizeof(z)));
  }
  return BI_OK;
}

int bi_selftest_wait_timeout(void* stream) {
  BI_RANGE("bi_selftest_wait_timeout");
  clear_error();
  BI_TRY(launch(wait_selftest_kernel, dim3(1), dim3(32), 0, as_stream(stream)));
  return BI_OK;
}

size_t bi_gemm_workspace_size(int M, int N, int K, int mode, int variant) {
  if (M <= 0 || N <= 0 || K <= 0 || N % 64 || K % 64) return 0;
  return gemm_ws_bytes(M, N, K, mode, variant);
}

int bi_gemm(const void* x, int ldx, const void* w, void* y, int ldy, int y_dtype, int M, int N, int K, int n_full,
            int epilogue, const bi_epi_args* epi, int mode, int variant, void* ws, size_t ws_bytes, void* stream) {
  BI_RANGE("bi_gemm");
  clear_error();
  return gemm_run(x, ldx, w, y, ldy, y_dtype, M, N, K, epilogue, epi, mode, variant, ws, ws_bytes, as_stream(stream),
                  n_full);
}

// early: the residual row and gamma were written before the kernel preceding
// this launch (the decode step's norms), so the kernel loads them before its
// dependency wait.
static int rmsnorm_run(const void* x, const void* residual_in, void* residual_out, const void* gamma, void* y,
                       float* y_f32, int M, int H, float eps, int mode, void* stream, bool early) {
  BI_REQUIRE(x && gamma && y, BI_ERR_INVALID_ARG, "bi_rmsnorm: NULL pointer");
  BI_REQUIRE(M >= 0 && H > 0 && H % 8 == 0 && H <= NORM_THREADS * NORM_MAX_CHUNKS * 8, BI_ERR_UNSUPPORTED,
             "bi_rmsnorm: H=%d (need H %% 8 == 0, H <= 16384)", H);
  BI_REQUIRE(mode_ok(mode), BI_ERR_INVALID_ARG, "bi_rmsnorm: bad mode");
  BI_REQUIRE(aligned16(x) && aligned16(gamma) && aligned16(y) && (!residual_in || aligned16(residual_in)) &&
                 (!residual_out || aligned16(residual_out)) && (!y_f32 || aligned16(y_f32)),
             BI_ERR_UNSUPPORTED, "bi_rmsnorm: buffers must be 16-byte aligned");
  if (M == 0) return BI_OK;
  const uint16_t* g16 = reinterpret_cast<const uint16_t*>(gamma);
  const int f32 = act_f32(mode), e = early ? 1 : 0;
  cudaStream_t st = as_stream(stream);
  switch (norm_cpt(H)) {
    case 1: return launch(rmsnorm_kernel<1>, dim3(M), dim3(NORM_THREADS), 0, st, x, residual_in, residual_out, g16, y,
                          y_f32, H, eps, f32, e);
    case 2: return launch(rmsnorm_kernel<2>, dim3(M), dim3(NORM_THREADS), 0, st, x, residual_in, residual_out, g16, y,
                          y_f32, H, eps, f32, e);
    case 4: return launch(rmsnorm_kernel<4>, dim3(M), dim3(NORM_THREADS), 0, st, x, residual_in, residual_out, g16, y,
                          y_f32, H, eps, f32, e);
    case 8: return launch(rmsnorm_kernel<8>, dim3(M), dim3(NORM_THREADS), 0, st, x, residual_in, residual_out, g16, y,
                          y_f32, H, eps, f32, e);
    default: return launch(rmsnorm_kernel<16>, dim3(M), dim3(NORM_THREADS), 0, st, x, residual_in, residual_out, g16,
                           y, y_f32, H, eps, f32, e);
  }
}

int bi_rmsnorm(const void* x, const void* residual_in, void* residual_out, const void* gamma, void* y, float* y_f32,
               int M, int H, float eps, int mode, void* stream) {
  BI_RANGE("bi_rmsnorm");
  clear_error();
  return rmsnorm_run(x, residual_in, residual_out, gamma, y, y_f32, M, H, eps, mode, stream, false);
}

int bi_rope_table_fill(float* table, int max_pos, int head_dim, double theta, void* stream) {
  BI_RANGE("bi_rope_table_fill");
  clear_error();
  BI_REQUIRE(table && max_pos > 0 && head_dim > 0 && head_dim % 2 == 0 && theta > 0, BI_ERR_INVALID_ARG,
             "bi_rope_table_fill: bad arguments");
  const int half = head_dim / 2;
  std::vector<float> host((size_t)max_pos * head_dim);
  for (int p = 0; p < max_pos; ++p)
    for (int i = 0; i < half; ++i) {
      const double ang = (double)p * std::pow(theta, -2.0 * i / head_dim);
      host[((size_t)p * half + i) * 2] = (float)std::cos(ang);
      host[((size_t)p * half + i) * 2 + 1] = (float)std::sin(ang);
    }
  // synchronous copy: the host buffer dies with this call
  BI_CHECK_CUDA(cudaStreamSynchronize(as_stream(stream)));
  BI_CHECK_CUDA(cudaMemcpy(table, host.data(), host.size() * sizeof(float), cudaMemcpyHostToDevice));
  return BI_OK;
}

int bi_rope_kv_append(const float* qkv, const float* rope, int rope_max_pos, void* q_out, const bi_kv_layout* kv,
                      int layer, const int32_t* slot, const int32_t* pos, int T, int Hq, int qk_paired, int mode,
                      void* stream) {
  BI_RANGE("bi_rope_kv_append");
  clear_error();
  BI_REQUIRE(qkv && rope && q_out && kv && kv->k && kv->v && slot && pos, BI_ERR_INVALID_ARG,
             "bi_rope_kv_append: NULL pointer");
  BI_REQUIRE(layer >= 0 && layer < kv->n_layers && T >= 0 && Hq > 0, BI_ERR_INVALID_ARG, "bi_rope_kv_append: bad args");
  BI_REQUIRE(mode_ok(mode) && kv->dtype == (act_f32(mode) ? BI_DTYPE_F32 : BI_DTYPE_BF16), BI_ERR_INVALID_ARG,
             "bi_rope_kv_append: KV dtype does not match the mode");
  if (T == 0) return BI_OK;
  BI_TRY(launch(rope_append_kernel, dim3(T), dim3(256), 0, as_stream(stream), qkv, rope, rope_max_pos, q_out, kv->k, kv->v, slot, pos, Hq,
                                                       kv->n_kv_heads, kv->head_dim, layer, kv->n_layers, kv->n_slots,
                                                       kv->capacity, act_f32(mode), qk_paired ? 1 : 0));
  return BI_OK;
}

size_t bi_attention_workspace_size(int T, int Hq, int head_dim, int max_pos) {
  if (T <= 0 || Hq <= 0 || head_dim <= 0 || max_pos < 0) return 0;
  // the largest of the invariant and FAST chunkings
  return std::max(std::max(attn_ws_bytes(T, Hq, head_dim, max_pos, 64), attn_ws_bytes(T, Hq, head_dim, max_pos, 128)),
                  attn_ws_bytes(T, Hq, head_dim, max_pos, 256));
}

int bi_attention(const void* q, const bi_kv_layout* kv, int layer, const int32_t* slot, const int32_t* pos,
                 const int32_t* slot_host, const int32_t* pos_host, void* out, int T, int Hq, float scale, int mode,
                 int variant, void* ws, size_t ws_bytes, void* stream) {
  BI_RANGE("bi_attention");
  clear_error();
  return attention_run(q, kv, layer, slot, pos, slot_host, pos_host, out, T, Hq, scale, mode, variant, ws, ws_bytes,
                       as_stream(stream));
}

size_t bi_lmhead_workspace_size(int B, int H, int V, int mode) {
  if (B <= 0 || H <= 0 || V <= 0) return 0;
  Carver cv(nullptr);
  lm_carve(cv, B, H, V, mode, true, lm_parts(mode, 1.f));
  return cv.used + 256;
}

int bi_lmhead_logprob(const float* h, const void* W, const int32_t* target, int B, int H, int V,
                      float margin_threshold, int mode, float* logprob, float* lse, int32_t* argmax, float* margin,
                      uint8_t* recomputed, float* logits, void* ws, size_t ws_bytes, void* stream) {
  BI_RANGE("bi_lmhead_logprob");
  clear_error();
  return lmhead_run(h, W, target, B, H, V, margin_threshold, mode, logprob, lse, argmax, margin, recomputed, logits,
                    ws, ws_bytes, as_stream(stream));
}

int bi_lmhead_split(const float* h, int B, int H, int parts, void* out, void* stream) {
  BI_RANGE("bi_lmhead_split");
  clear_error();
  BI_REQUIRE(h && out && B >= 0 && H > 0 && (parts == 1 || parts == 3), BI_ERR_INVALID_ARG,
             "bi_lmhead_split: bad arguments");
  if (B == 0) return BI_OK;
  const size_t n = (size_t)B * H;
  BI_TRY(launch(lm_split_kernel, dim3((int)std::min<size_t>((n + 255) / 256, 4096)), dim3(256), 0, as_stream(stream),
                h, reinterpret_cast<uint16_t*>(out), n, parts));
  return BI_OK;
}

size_t bi_lmhead_logits_workspace_size(int B, int V) {
  if (B <= 0 || V <= 0) return 0;
  Carver cv(nullptr);
  lm_stage_carve(cv, B, V);
  return cv.used + 256;
}

int bi_lmhead_from_logits(const float* z, int B, int V, int parts, const int32_t* target, float margin_threshold,
                          float* logprob, float* lse, int32_t* argmax, float* margin, uint8_t* recomputed, void* ws,
                          size_t ws_bytes, void* stream) {
  BI_RANGE("bi_lmhead_from_logits");
  clear_error();
  return lm_from_logits_run(z, B, V, parts, target, margin_threshold, logprob, lse, argmax, margin, recomputed, ws,
                            ws_bytes, as_stream(stream));
}

int bi_ctx_create(const bi_model_desc* desc, const bi_weights* w, const bi_kv_layout* kv, bi_ctx** out) {
  clear_error();
  BI_REQUIRE(desc && w && kv && out, BI_ERR_INVALID_ARG, "bi_ctx_create: NULL pointer");
  const bi_model_desc& d = *desc;
  BI_REQUIRE(d.n_layers > 0 && d.hidden > 0 && d.n_heads > 0 && d.n_kv_heads > 0 && d.head_dim > 0 && d.ffn > 0 &&
                 d.vocab > 0,
             BI_ERR_INVALID_ARG, "bi_ctx_create: bad model sizes");
  BI_REQUIRE(d.n_heads % d.n_kv_heads == 0, BI_ERR_INVALID_ARG, "bi_ctx_create: n_heads %% n_kv_heads != 0");
  BI_REQUIRE(mode_ok(d.mode), BI_ERR_INVALID_ARG, "bi_ctx_create: bad mode");
  BI_REQUIRE(d.variant == BI_VARIANT_INVARIANT || d.variant == BI_VARIANT_FAST, BI_ERR_INVALID_ARG,
             "bi_ctx_create: bad variant");
  const int QKV = (d.n_heads + 2 * d.n_kv_heads) * d.head_dim;
  BI_REQUIRE(d.hidden % 64 == 0 && d.ffn % 64 == 0 && d.vocab % 64 == 0 && QKV % 64 == 0 &&
                 (d.n_heads * d.head_dim) % 64 == 0 && d.ffn % BI_GU_INTERLEAVE == 0,
             BI_ERR_UNSUPPORTED, "bi_ctx_create: hidden/ffn/vocab/projection sizes must be multiples of 64");
  BI_REQUIRE(d.head_dim == 64 || d.head_dim == 128, BI_ERR_UNSUPPORTED, "bi_ctx_create: head_dim must be 64 or 128");
  BI_REQUIRE(d.hidden <= 16384, BI_ERR_UNSUPPORTED, "bi_ctx_create: hidden > 16384");
  BI_REQUIRE(d.n_heads / d.n_kv_heads <= ATT_MAX_PAIRS, BI_ERR_UNSUPPORTED,
             "bi_ctx_create: %d q heads per kv head (max %d)", d.n_heads / d.n_kv_heads, ATT_MAX_PAIRS);
  BI_REQUIRE(w->embed && w->lm_head && w->final_norm && w->attn_norm && w->ffn_norm && w->w_qkv && w->w_o &&
                 w->w_gu && w->w_down && w->rope && w->rope_max_pos > 0,
             BI_ERR_INVALID_ARG, "bi_ctx_create: NULL weight pointer");
  BI_REQUIRE(kv->k && kv->v && kv->n_layers == d.n_layers && kv->n_kv_heads == d.n_kv_heads &&
                 kv->head_dim == d.head_dim && kv->n_slots > 0 && kv->capacity > 0,
             BI_ERR_INVALID_ARG, "bi_ctx_create: KV layout does not match the model");
  BI_REQUIRE(kv->dtype == (act_f32(d.mode) ? BI_DTYPE_F32 : BI_DTYPE_BF16), BI_ERR_INVALID_ARG,
             "bi_ctx_create: KV dtype does not match the mode");
  bi_ctx* c = new (std::nothrow) bi_ctx;
  BI_REQUIRE(c, BI_ERR_INVALID_ARG, "bi_ctx_create: out of host memory");
  c->desc = d;
  c->w = *w;
  c->kv = *kv;
  *out = c;
  return BI_OK;
}

int bi_ctx_destroy(bi_ctx* ctx) {
  delete ctx;
  return BI_OK;
}

struct StepWs {
  void *res, *u, *y, *q, *o, *a;
  float* qkv;
  float* h32;
  float* hl;
  uint8_t* attn;
  size_t attn_bytes;
  uint8_t* lm;
  size_t lm_bytes;
  uint8_t* gemm;  // split-K partials of the FAST variant
  size_t gemm_bytes;
};

static StepWs step_carve(Carver& cv, const bi_model_desc& d, int T, int n_lm, int max_pos) {
  const size_t es = act_f32(d.mode) ? 4 : 2;
  const int QD = d.n_heads * d.head_dim, KD = d.n_kv_heads * d.head_dim;
  StepWs s{};
  s.res = cv.take<uint8_t>((size_t)T * d.hidden * es);
  s.u = cv.take<uint8_t>((size_t)T * d.hidden * es);
  s.y = cv.take<uint8_t>((size_t)T * d.hidden * es);
  s.q = cv.take<uint8_t>((size_t)T * QD * es);
  s.o = cv.take<uint8_t>((size_t)T * QD * es);
  s.a = cv.take<uint8_t>((size_t)T * d.ffn * es);
  s.qkv = cv.take<float>((size_t)T * (QD + 2 * KD));
  s.h32 = cv.take<float>((size_t)T * d.hidden);
  s.hl = cv.take<float>((size_t)std::max(n_lm, 1) * d.hidden);
  s.attn_bytes = bi_attention_workspace_size(T, d.n_heads, d.head_dim, max_pos);
  s.attn = cv.take<uint8_t>(s.attn_bytes);
  s.lm_bytes = bi_lmhead_workspace_size(std::max(n_lm, 1), d.hidden, d.vocab, d.mode);
  s.lm = cv.take<uint8_t>(s.lm_bytes);
  const int QKV = QD + 2 * KD;
  s.gemm_bytes = std::max(std::max(gemm_ws_bytes(T, QKV, d.hidden, d.mode, d.variant),
                                   gemm_ws_bytes(T, d.hidden, QD, d.mode, d.variant)),
                          std::max(gemm_ws_bytes(T, 2 * d.ffn, d.hidden, d.mode, d.variant),
                                   gemm_ws_bytes(T, d.hidden, d.ffn, d.mode, d.variant)));
  s.gemm = s.gemm_bytes ? cv.take<uint8_t>(s.gemm_bytes) : nullptr;
  return s;
}

size_t bi_decode_workspace_size(const bi_ctx* ctx, int max_tokens, int max_lm_rows, int max_pos) {
  if (!ctx || max_tokens <= 0 || max_lm_rows < 0 || max_pos < 0) return 0;
  Carver cv(nullptr);
  step_carve(cv, ctx->desc, max_tokens, max_lm_rows, max_pos);
  return cv.used + 256;
}

__global__ void gather_lm_rows_kernel(const int32_t* __restrict__ lm_row, const float* __restrict__ h32, int T, int H,
                                      int n_lm, float* __restrict__ hl, float* __restrict__ h_out) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  const int r = lm_row[t];
  if (r < 0) return;
  if (r >= n_lm) {
    if (threadIdx.x == 0) dev_flag(DEVERR_INDEX);
    return;
  }
  for (int i = threadIdx.x; i < H; i += blockDim.x) {
    const float v = h32[(size_t)t * H + i];
    hl[(size_t)r * H + i] = v;
    if (h_out) h_out[(size_t)r * H + i] = v;
  }
}

int bi_decode_step(bi_ctx* ctx, const bi_batch* batch, const bi_step_out* out, void* ws, size_t ws_bytes,
                   void* stream) {
  BI_RANGE("bi_decode_step");
  clear_error();
  BI_REQUIRE(ctx && batch && out, BI_ERR_INVALID_ARG, "bi_decode_step: NULL pointer");
  const bi_model_desc& d = ctx->desc;
  const bi_weights& w = ctx->w;
  const int T = batch->n_tokens, n_lm = batch->n_lm;
  BI_REQUIRE(T >= 0 && n_lm >= 0 && n_lm <= T, BI_ERR_INVALID_ARG, "bi_decode_step: n_tokens=%d n_lm=%d", T, n_lm);
  if (T == 0) return BI_OK;
  BI_REQUIRE(batch->ids && batch->slot && batch->pos && batch->slot_host && batch->pos_host && batch->lm_row,
             BI_ERR_INVALID_ARG, "bi_decode_step: NULL batch array");
  BI_REQUIRE(n_lm == 0 || (out->logprob && out->lse && out->argmax && out->margin && out->recomputed),
             BI_ERR_INVALID_ARG, "bi_decode_step: NULL output array");
  int max_pos = 0;
  for (int t = 0; t < T; ++t) {  // every host-checkable argument is checked before the first launch
    const int sl = batch->slot_host[t], p = batch->pos_host[t];
    BI_REQUIRE(sl >= 0 && sl < ctx->kv.n_slots, BI_ERR_INVALID_ARG, "bi_decode_step: token %d slot %d of %d", t, sl,
               ctx->kv.n_slots);
    BI_REQUIRE(p >= 0 && p < ctx->kv.capacity && p < w.rope_max_pos, BI_ERR_CAPACITY,
               "bi_decode_step: token %d position %d beyond KV capacity %d / RoPE table %d", t, p, ctx->kv.capacity,
               w.rope_max_pos);
    max_pos = std::max(max_pos, p);
  }
  const size_t need = bi_decode_workspace_size(ctx, T, n_lm, max_pos);
  BI_REQUIRE(ws && ws_bytes >= need, BI_ERR_WORKSPACE, "bi_decode_step: workspace %zu < %zu", ws_bytes, need);
  Carver cv(reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255)));
  StepWs s = step_carve(cv, d, T, n_lm, max_pos);
  cudaStream_t st = as_stream(stream);
  const int H = d.hidden, Hq = d.n_heads, Hkv = d.n_kv_heads, hd = d.head_dim, F = d.ffn;
  const int QD = Hq * hd, KD = Hkv * hd, QKV = QD + 2 * KD;
  const int f32 = act_f32(d.mode);
  const int act_dtype = f32 ? BI_DTYPE_F32 : BI_DTYPE_BF16;
  const size_t wbytes = d.mode == BI_MODE_FP32 ? 4 : 2;  // projection weights; the norm gains are bf16 in every mode
  const float scale = 1.0f / std::sqrt((float)hd);
  auto lw = [&](const void* base, size_t per_layer, int l) {
    return reinterpret_cast<const void*>(reinterpret_cast<const uint8_t*>(base) + per_layer * l * wbytes);
  };
  auto lg = [&](const void* base, int l) {  // per-layer norm gain (bf16)
    return reinterpret_cast<const void*>(reinterpret_cast<const uint8_t*>(base) + (size_t)H * l * 2);
  };

  if (d.mode == BI_MODE_FP32)
    BI_TRY(launch(embed_kernel<float>, dim3(T), dim3(256), 0, st, batch->ids, reinterpret_cast<const float*>(w.embed),
                  s.y, H, d.vocab, f32));
  else
    BI_TRY(launch(embed_kernel<uint16_t>, dim3(T), dim3(256), 0, st, batch->ids,
                  reinterpret_cast<const uint16_t*>(w.embed), s.y, H, d.vocab, f32));
  for (int l = 0; l < d.n_layers; ++l) {
    const void* g_attn = lg(w.attn_norm, l);
    const void* g_ffn = lg(w.ffn_norm, l);
    // the step's norms read the residual row written by the norm two or more kernels back (early loads)
    BI_TRY(rmsnorm_run(s.y, l == 0 ? nullptr : s.res, s.res, g_attn, s.u, nullptr, T, H, d.eps, d.mode, stream,
                       true));
    if (f32 || d.variant == BI_VARIANT_FAST) {  // projection, then RoPE + KV append as a kernel
      BI_TRY(gemm_run(s.u, H, lw(w.w_qkv, (size_t)QKV * H, l), s.qkv, QKV, BI_DTYPE_F32, T, QKV, H, BI_EPI_NONE,
                      nullptr, d.mode, d.variant, s.gemm, s.gemm_bytes, st));
      BI_TRY(bi_rope_kv_append(s.qkv, w.rope, w.rope_max_pos, s.q, &ctx->kv, l, batch->slot, batch->pos, T, Hq, 1,
                               d.mode, stream));
    } else {  // RoPE + KV append in the projection's epilogue
      const bi_epi_args ea{w.rope, w.rope_max_pos, s.q, &ctx->kv, l, batch->slot, batch->pos, Hq};
      BI_TRY(gemm_run(s.u, H, lw(w.w_qkv, (size_t)QKV * H, l), nullptr, QKV, BI_DTYPE_BF16, T, QKV, H,
                      BI_EPI_ROPE_KV_APPEND, &ea, d.mode, d.variant, nullptr, 0, st));
    }
    BI_TRY(attention_run(s.q, &ctx->kv, l, batch->slot, batch->pos, batch->slot_host, batch->pos_host, s.o, T, Hq,
                         scale, d.mode, d.variant, s.attn, s.attn_bytes, st, true));
    BI_TRY(gemm_run(s.o, QD, lw(w.w_o, (size_t)H * QD, l), s.y, H, act_dtype, T, H, QD, BI_EPI_NONE, nullptr, d.mode,
                    d.variant, s.gemm, s.gemm_bytes, st));
    BI_TRY(rmsnorm_run(s.y, s.res, s.res, g_ffn, s.u, nullptr, T, H, d.eps, d.mode, stream, true));
    BI_TRY(gemm_run(s.u, H, lw(w.w_gu, (size_t)2 * F * H, l), s.a, F, act_dtype, T, 2 * F, H, BI_EPI_SWIGLU, nullptr, d.mode,
                    d.variant, s.gemm, s.gemm_bytes, st));
    BI_TRY(gemm_run(s.a, F, lw(w.w_down, (size_t)H * F, l), s.y, H, act_dtype, T, H, F, BI_EPI_NONE, nullptr, d.mode,
                    d.variant, s.gemm, s.gemm_bytes, st));
  }
  BI_TRY(rmsnorm_run(s.y, s.res, s.res, w.final_norm, s.u, s.h32, T, H, d.eps, d.mode, stream, true));
  if (n_lm == 0) return BI_OK;
  BI_TRY(launch(gather_lm_rows_kernel, dim3(T), dim3(256), 0, st, batch->lm_row, s.h32, T, H, n_lm, s.hl, out->h));
  return lmhead_run(s.hl, w.lm_head, batch->target, n_lm, H, d.vocab, d.margin_threshold, d.mode, out->logprob,
                    out->lse, out->argmax, out->margin, out->recomputed, out->logits, s.lm, s.lm_bytes, st);
}

// ------------------------------------------------ LM head without caller-supplied scratch
// Some callers cannot call cudaMalloc: code that runs while a caching
// allocator owns all device memory, plug-ins that are handed only their
// inputs and outputs, or hosts that forbid allocation on the request path.
// For them bi_lmhead_logprob_noalloc takes its scratch from this fixed
// file-scope array instead of a workspace argument.  The array is part of
// the library image: every GPU that loads the library holds it until the
// process exits.
static __device__ __align__(256) uint8_t g_noalloc_scratch[BI_NOALLOC_SCRATCH_BYTES];

// Device address of the array on each device.  Host code cannot use the
// symbol itself (on the host it names a stand-in, not device memory), so the
// address is looked up once per device, with that device current, and kept
// for the life of the process (a device reset invalidates it; the header
// tells callers not to use this entry point after one).
static int noalloc_scratch_ptr(void** out) {
  static std::mutex mu;
  static std::vector<void*> addr;
  int dev = 0;
  BI_CHECK_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> g(mu);
  if ((int)addr.size() <= dev) addr.resize(dev + 1, nullptr);
  if (!addr[dev]) {
    void* p = nullptr;
    BI_CHECK_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    addr[dev] = p;
  }
  *out = addr[dev];
  return BI_OK;
}

int bi_lmhead_logprob_noalloc(const float* h, const void* W, const int32_t* target, int B, int H, int V,
                              float margin_threshold, int mode, float* logprob, float* lse, int32_t* argmax,
                              float* margin, uint8_t* recomputed, float* logits, void* stream) {
  BI_RANGE("bi_lmhead_logprob_noalloc");
  clear_error();
  BI_REQUIRE(B >= 0 && H > 0 && V > 0, BI_ERR_INVALID_ARG, "bi_lmhead_logprob_noalloc: bad sizes");
  if (B == 0) return BI_OK;
  Carver probe(nullptr);
  lm_carve(probe, B, H, V, mode, logits == nullptr, lm_parts(mode, margin_threshold));
  const size_t need = probe.used + 256;
  BI_REQUIRE(need <= (size_t)BI_NOALLOC_SCRATCH_BYTES, BI_ERR_WORKSPACE,
             "bi_lmhead_logprob_noalloc: B=%d H=%d V=%d needs %zu bytes of scratch, more than the fixed %d; "
             "use bi_lmhead_logprob with a workspace or fewer rows",
             B, H, V, need, BI_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  BI_TRY(noalloc_scratch_ptr(&scratch));
  // Every scratch byte the kernels read is written earlier in the same call,
  // so nothing needs clearing between calls.
  return lmhead_run(h, W, target, B, H, V, margin_threshold, mode, logprob, lse, argmax, margin, recomputed, logits,
                    scratch, BI_NOALLOC_SCRATCH_BYTES, as_stream(stream));
}

int bi_embed(const int32_t* ids, const void* embed, int T, int H, int V, int mode, void* x, void* stream) {
  BI_RANGE("bi_embed");
  clear_error();
  BI_REQUIRE(ids && embed && x && T >= 0 && H > 0 && V > 0, BI_ERR_INVALID_ARG, "bi_embed: bad arguments");
  BI_REQUIRE(mode_ok(mode), BI_ERR_INVALID_ARG, "bi_embed: bad mode");
  if (T == 0) return BI_OK;
  if (mode == BI_MODE_FP32)
    BI_TRY(launch(embed_kernel<float>, dim3(T), dim3(256), 0, as_stream(stream), ids,
                  reinterpret_cast<const float*>(embed), x, H, V, 1));
  else
    BI_TRY(launch(embed_kernel<uint16_t>, dim3(T), dim3(256), 0, as_stream(stream), ids,
                  reinterpret_cast<const uint16_t*>(embed), x, H, V, act_f32(mode)));
  return BI_OK;
}

int bi_greedy_advance(const int32_t* argmax, int32_t* ids, int32_t* pos, int B, void* stream) {
  BI_RANGE("bi_greedy_advance");
  clear_error();
  BI_REQUIRE(argmax && ids && pos && B >= 0, BI_ERR_INVALID_ARG, "bi_greedy_advance: bad arguments");
  if (B == 0) return BI_OK;
  BI_TRY(launch(greedy_advance_kernel, dim3((B + 127) / 128), dim3(128), 0, as_stream(stream), argmax, ids, pos, B));
  return BI_OK;
}

int bi_synth_fill_bf16(uint16_t* dst, int64_t rows, int64_t cols, uint64_t key, double std, int interleave, int phase,
                       void* stream) {
  BI_RANGE("bi_synth_fill_bf16");
  clear_error();
  BI_REQUIRE(dst && rows >= 0 && cols > 0 && (phase == 0 || phase == 1), BI_ERR_INVALID_ARG,
             "bi_synth_fill_bf16: bad arguments");
  BI_REQUIRE(interleave >= 0 || interleave == -64 || interleave == -128, BI_ERR_INVALID_ARG,
             "bi_synth_fill_bf16: paired order needs head_dim 64 or 128");
  BI_REQUIRE(interleave == 0 || rows % (interleave > 0 ? interleave : -interleave) == 0, BI_ERR_INVALID_ARG,
             "bi_synth_fill_bf16: rows must be a multiple of the interleave");
  if (rows == 0) return BI_OK;
  BI_TRY(launch(synth_fill_kernel, dim3(4 * num_sms()), dim3(256), 0, as_stream(stream), dst, rows, cols, key, std, interleave, phase));
  return BI_OK;
}

}  // extern "C"
