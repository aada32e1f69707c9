// bi_gemm: launch planning for the tcgen05 GEMM (gemm_tc.cuh), the FAST
// variant's split-K reduction, and the LayerCast routes.
//
// Invariance ("Meituan bitwise train/infer consistency": full-K computation in
// place of segmented reductions, one accumulation order for Prefill and
// Decode): every output element y[m][n] is accumulated in fp32 over the full K
// range, in ascending K, by the same instruction sequence whatever M is (the
// tcgen05 kernel's header states the argument).  The launch shape -- weight
// tile, token tiles per weight stage, token rows staged, CTAs per SM -- is
// chosen here from M and N for speed; it is work assignment only.
//
// LayerCast ("Give Me FP32 or Give Me Death?", LayerCast section: bf16-stored
// weights, fp32 arithmetic): every projection and the LM head
// (gemm_layercast, at the end of this file) split each f32 activation exactly
// into three bf16 parts and run them through the invariant tensor-core GEMM.
// The FP32-storage mode (f32 weights) takes every product and sum as an fp32
// FMA (gemm_f32_kernel).  Element order there: lane l of a warp owns the
// k-slices [256 i + 8 l, 256 i + 8 l + 8) for i = 0, 1, ...; it accumulates
// them with sequential FMAs in ascending k, and the 32 lane partials are then
// combined by a fixed xor-butterfly.  This is the same for every M and every
// row/token tiling.
#pragma once
#include <algorithm>

#include "common.cuh"
#include "gemm_tc.cuh"
#include "gemm_mma.cuh"

namespace bi {

// ---------------------------------------------------------------- LayerCast (fp32 FMA)
constexpr int F32_ROWS = 32;  // weight rows per CTA (8 warps x 4 rows)
constexpr int F32_TOK = 16;   // token columns per CTA
constexpr int F32_KC = 256;   // k per chunk (32 lanes x 8)

// x: f32 [M][ldx]; w: [N][K], bf16 (WT = uint16_t, upcast in registers) or
// f32 (WT = float: the FP32-storage mode); y: [M][ldy].  Optional device row
// count (count != nullptr): only token rows < *count are computed (used by the
// selective recompute, whose row count is known only on the device).
// The CTA's 16 token rows are staged chunk by chunk (256 k) in shared memory,
// double-buffered, and read by all 8 warps; each warp streams 4 weight rows.
// The weight type changes only how 8 weights are fetched, not the FMA order.
template <int EPI, typename WT>
__global__ void __launch_bounds__(256)
    gemm_f32_kernel(const float* __restrict__ x, int ldx, const WT* __restrict__ w, void* __restrict__ y,
                    int ldy, int y_f32, int M, int N, int K, const int* __restrict__ count) {
  pdl_wait();
  pdl_trigger();
  __shared__ __align__(16) float xs[2][F32_TOK][F32_KC];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * F32_TOK;
  int Meff = M;
  if (count) Meff = min(M, *count);
  if (m0 >= Meff) return;
  const int ntok = min(F32_TOK, Meff - m0);
  const int grp = blockIdx.y;
  int rows[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    if constexpr (EPI == BI_EPI_SWIGLU)
      rows[r] = grp * F32_ROWS + (r >> 1) * 16 + 2 * warp + (r & 1);  // 2 gate rows, then the 2 matching up rows
    else
      rows[r] = grp * F32_ROWS + 4 * warp + r;
  }
  // staging: thread t copies 16 consecutive floats of token t / 16 at offset (t % 16) * 16
  const int st_tok = threadIdx.x >> 4, st_off = (threadIdx.x & 15) * 16;
  auto fetch = [&](int kc, float4* v) {
    const int k = kc * F32_KC + st_off;
    const bool ok = st_tok < ntok && k < K;
    const float4* src = reinterpret_cast<const float4*>(x + (size_t)(m0 + st_tok) * ldx + k);
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = ok ? __ldg(src + q) : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  auto stash = [&](int buf, const float4* v) {
    float4* dst = reinterpret_cast<float4*>(&xs[buf][st_tok][st_off]);
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = v[q];
  };
  float acc[4][F32_TOK];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int t = 0; t < F32_TOK; ++t) acc[r][t] = 0.f;

  const int nk = (K + F32_KC - 1) / F32_KC;
  {
    float4 v[4];
    fetch(0, v);
    stash(0, v);
  }
  __syncthreads();
  for (int kc = 0; kc < nk; ++kc) {
    const int buf = kc & 1;
    float4 nxt[4];
    if (kc + 1 < nk) fetch(kc + 1, nxt);
    const int k = kc * F32_KC + 8 * lane;
    if (k < K) {
      float wv8[4][8];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        if constexpr (sizeof(WT) == 2) {
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(w + (size_t)rows[r] * K + k));
          const uint32_t words[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int j = 0; j < 8; ++j) wv8[r][j] = (j & 1) ? bf16hi(words[j >> 1]) : bf16lo(words[j >> 1]);
        } else {
          const float4 a = __ldg(reinterpret_cast<const float4*>(w + (size_t)rows[r] * K + k));
          const float4 b = __ldg(reinterpret_cast<const float4*>(w + (size_t)rows[r] * K + k + 4));
          wv8[r][0] = a.x; wv8[r][1] = a.y; wv8[r][2] = a.z; wv8[r][3] = a.w;
          wv8[r][4] = b.x; wv8[r][5] = b.y; wv8[r][6] = b.z; wv8[r][7] = b.w;
        }
      }
#pragma unroll
      for (int t = 0; t < F32_TOK; ++t) {
        if (t < ntok) {
          const float4 x0 = *reinterpret_cast<const float4*>(&xs[buf][t][8 * lane]);
          const float4 x1 = *reinterpret_cast<const float4*>(&xs[buf][t][8 * lane + 4]);
          const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
#pragma unroll
            for (int r = 0; r < 4; ++r) acc[r][t] = fmaf(wv8[r][j], xv[j], acc[r][t]);
          }
        }
      }
    }
    if (kc + 1 < nk) stash(buf ^ 1, nxt);
    __syncthreads();
  }
#pragma unroll
  for (int t = 0; t < F32_TOK; ++t) {
    if (t >= ntok) break;
    float sr[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) sr[r] = warp_sum_fixed(acc[r][t]);
    const int m = m0 + t;
    if constexpr (EPI == BI_EPI_SWIGLU) {
      if (lane < 2) {
        const float gv = lane == 0 ? sr[0] : sr[1];
        const float uv = lane == 0 ? sr[2] : sr[3];
        const int col = grp * 16 + 2 * warp + lane;
        store_act(y, (size_t)m * ldy + col, silu(gv) * uv, y_f32);
      }
    } else {
#pragma unroll
      for (int r = 0; r < 4; ++r)
        if (lane == r) store_act(y, (size_t)m * ldy + rows[r], sr[r], y_f32);
    }
  }
}

// ---------------------------------------------------------------- host side
// Split factor of the FAST variant: more K splits for small M so that the
// grid fills the SMs (the usual library heuristic) -- which is exactly what
// makes the result depend on the batch size.
static int gemm_fast_splits(int M, int n_items, int kstages) {
  const int sms = num_sms();
  if (M > 16) return 1;
  int s = (2 * sms + n_items - 1) / n_items;
  if (M <= 4) s *= 2;
  s = s < 1 ? 1 : (s > 8 ? 8 : s);
  while (s > 1 && kstages / s < 2) --s;
  return s;
}

// Launch shape of the tcgen05 GEMM (work assignment only; see gemm_tc.cuh for
// why none of it changes an element's bits).  KS accumulator sets of BN x MT
// columns must fit the 512 TMEM columns.
struct TcPlan {
  int bn, mt, ks, splits;
};
constexpr int TC_XR = 128;  // token rows staged per tile (launches of more than 32 rows)
static int tc_kbs(int bn, int mt) {
  const int kb = (bn + mt * TC_XR) * 128;
  return kb <= 8192 ? 4 : (kb <= 24576 ? 2 : 1);
}
static TcPlan tc_plan(int M, int N, int K, int variant, int ks) {
  TcPlan p{};
  p.ks = ks;
  p.mt = (M <= TC_TILE_M || p.ks == 4) ? 1 : 2;
  // widest weight tile the TMEM holds (one token tile: at most 128 rows, so that
  // the launches of up to 128 tokens spread over more SMs); four-set matrices
  // take 64-row tiles when 128-row ones would leave SMs without an item (the
  // launch is then bound by the weight stream, e.g. LayerCast's split rows)
  int cols = std::min(512 / (p.ks * p.mt), p.mt == 1 ? 128 : 256);
  if (p.ks == 4 && (N / 128) * ((M + TC_TILE_M - 1) / TC_TILE_M) < num_sms()) cols = 64;
  p.bn = (cols >= 256 && N % 256 == 0) ? 256 : ((cols >= 128 && N % 128 == 0) ? 128 : 64);
  p.splits = 1;
  if (variant == BI_VARIANT_FAST) {
    const int items = (N / p.bn) * ((M + p.mt * TC_TILE_M - 1) / (p.mt * TC_TILE_M));
    const int kbs = tc_kbs(p.bn, p.mt);
    p.splits = gemm_fast_splits(M, items, (K / TC_BK + kbs - 1) / kbs);
  }
  return p;
}
// Launches of at most this many token rows run on the mma.sync kernel, whose
// 32-row weight tiles spread the small projections of a decode step over every
// SM; larger ones on tcgen05, whose 128-row MMA is then filled.
constexpr int MMA_MAX_ROWS = 32;

// LayerCast on tensor cores: rows of x per pass (bounds the workspace)
constexpr int LC_ROWS = 256;
// col_block > 0: the output columns are computed col_block at a time (a
// multiple of 256), so the workspace holds one block's three partial products.
static size_t lc_ws_bytes(int M, int N, int K, int col_block = 0) {
  const size_t mb = (size_t)std::min(M, LC_ROWS);
  const size_t nb = (size_t)(col_block > 0 ? std::min(N, col_block) : N);
  return 3 * mb * K * 2 + 3 * mb * nb * 4 + 512;
}

size_t gemm_ws_bytes(int M, int N, int K, int mode, int variant) {
  if (mode == BI_MODE_LAYERCAST) return M > 0 ? lc_ws_bytes(M, N, K) : 0;
  if (variant != BI_VARIANT_FAST || M <= 0) return 0;
  int splits;
  if (M <= MMA_MAX_ROWS) {
    const int bn = gemm_pick_bn(N), kbs = gemm_kbs(bn);
    splits = gemm_fast_splits(M, (N / bn) * ((M + GEMM_BM - 1) / GEMM_BM), (K / GEMM_BK + kbs - 1) / kbs);
  } else {
    splits = tc_plan(M, N, K, variant, gemm_ks(N)).splits;
  }
  return splits > 1 ? (size_t)splits * M * N * sizeof(float) : 0;
}

template <int BN, int MT, int KS, int EPI>
static int launch_tc_t(const CUtensorMap& tw, const CUtensorMap& tx, const TcArgs& a, cudaStream_t st) {
  using C = TcCfg<BN, MT, TC_XR, KS, 1>;
  static bool attr_done = false;  // per instantiation; set once per process
  if (!attr_done) {
    BI_CHECK_CUDA(cudaFuncSetAttribute(gemm_tc_kernel<BN, MT, TC_XR, KS, EPI, 1>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
    attr_done = true;
  }
  const int items = a.splits * a.n_groups * a.m_groups;
  const int grid = items < num_sms() ? items : num_sms();
  BI_TRY(launch(gemm_tc_kernel<BN, MT, TC_XR, KS, EPI, 1>, dim3(grid), dim3(TC_THREADS), C::SMEM, st, tw, tx, a));
  return BI_OK;
}

template <int EPI>
static int launch_tc_epi(const TcPlan& p, const CUtensorMap& tw, const CUtensorMap& tx, const TcArgs& a,
                         cudaStream_t st) {
#define BI_TC_CASE(BNV, MTV, KSV) \
  if (p.bn == BNV && p.mt == MTV && p.ks == KSV) return launch_tc_t<BNV, MTV, KSV, EPI>(tw, tx, a, st);
  BI_TC_CASE(256, 2, 1)
  BI_TC_CASE(128, 2, 1)
  BI_TC_CASE(64, 2, 1)
  BI_TC_CASE(128, 1, 1)
  BI_TC_CASE(64, 1, 1)
  BI_TC_CASE(128, 2, 2)
  BI_TC_CASE(64, 2, 2)
  BI_TC_CASE(128, 1, 2)
  BI_TC_CASE(64, 1, 2)
  BI_TC_CASE(128, 1, 4)
  BI_TC_CASE(64, 1, 4)
#undef BI_TC_CASE
  return set_error(BI_ERR_UNSUPPORTED, "bi_gemm: no tcgen05 kernel for tile %d x %d with %d accumulator sets", p.bn,
                   p.mt, p.ks);
}

static int gemm_tc(const void* x, int ldx, const void* w, void* y, int ldy, int y_f32, int M, int N, int K, int epi,
                   int ks, int variant, void* ws, size_t ws_bytes, cudaStream_t st, const int* mcount, int mmult,
                   const RopeEpi* rope) {
  const TcPlan p = tc_plan(M, N, K, variant, ks);
  const int kbs = tc_kbs(p.bn, p.mt);
  // 3-D views {64 k, rows, k-block}: the k-block dimension (stride 128 B) is the
  // outermost of the box, so a box lands as kbs swizzled [rows][128 B] slabs.
  CUtensorMap tw, tx;
  const uint64_t dw[3] = {(uint64_t)TC_BK, (uint64_t)N, (uint64_t)(K / TC_BK)};
  const uint64_t sw[2] = {(uint64_t)K * 2, (uint64_t)TC_BK * 2};
  const uint32_t bw[3] = {(uint32_t)TC_BK, (uint32_t)p.bn, (uint32_t)kbs};
  BI_TRY(encode_tmap_3d(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w, dw, sw, bw, CU_TENSOR_MAP_SWIZZLE_128B));
  const uint64_t dx[3] = {(uint64_t)TC_BK, (uint64_t)M, (uint64_t)(K / TC_BK)};
  const uint64_t sx[2] = {(uint64_t)ldx * 2, (uint64_t)TC_BK * 2};
  const uint32_t bx[3] = {(uint32_t)TC_BK, (uint32_t)(TC_XR * p.mt), (uint32_t)kbs};
  BI_TRY(encode_tmap_3d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, dx, sx, bx, CU_TENSOR_MAP_SWIZZLE_128B));
  TcArgs a{};
  a.y = y;
  a.ldy = ldy;
  a.y_f32 = y_f32;
  a.vec_ok = (reinterpret_cast<uintptr_t>(y) % 16 == 0) && ((size_t)ldy * (y_f32 ? 4 : 2)) % 16 == 0;
  a.M = M;
  a.N = N;
  a.K = K;
  a.m_groups = (M + p.mt * TC_TILE_M - 1) / (p.mt * TC_TILE_M);
  a.n_groups = N / p.bn;
  // token rows of a band of the work order: about 48 MB, so that a band stays in L2
  const size_t group_bytes = (size_t)p.mt * TC_TILE_M * K * 2;
  a.m_band = (int)std::max<size_t>(1, std::min<size_t>(a.m_groups, (size_t(48) << 20) / group_bytes));
  a.splits = p.splits;
  a.mcount = mcount;
  a.mmult = mmult;
  if (rope) a.re = *rope;
  if (p.splits > 1) {
    const size_t need = (size_t)p.splits * M * N * sizeof(float);
    BI_REQUIRE(ws && ws_bytes >= need, BI_ERR_WORKSPACE, "bi_gemm FAST: workspace %zu < %zu", ws_bytes, need);
    a.partial = reinterpret_cast<float*>(ws);
  }
  if (epi == EPI_ROPE) {
    if (p.splits > 1 || !rope) return set_error(BI_ERR_UNSUPPORTED, "fused RoPE epilogue needs one split and its table");
    BI_TRY(launch_tc_epi<EPI_ROPE>(p, tw, tx, a, st));
  } else if (epi == BI_EPI_SWIGLU) {
    BI_TRY(launch_tc_epi<BI_EPI_SWIGLU>(p, tw, tx, a, st));
  } else {
    BI_TRY(launch_tc_epi<BI_EPI_NONE>(p, tw, tx, a, st));
  }
  if (p.splits > 1) {
    const int n_out = epi == BI_EPI_SWIGLU ? N / 2 : N;
    const size_t total = (size_t)M * n_out;
    int blocks = (int)((total + 255) / 256);
    if (blocks > 4 * num_sms()) blocks = 4 * num_sms();
    if (epi == BI_EPI_SWIGLU)
      BI_TRY(launch(splitk_reduce_kernel<BI_EPI_SWIGLU>, dim3(blocks), dim3(256), 0, st, a.partial, y, ldy, y_f32, M, N,
                    p.splits));
    else
      BI_TRY(launch(splitk_reduce_kernel<BI_EPI_NONE>, dim3(blocks), dim3(256), 0, st, a.partial, y, ldy, y_f32, M, N,
                    p.splits));
  }
  return BI_OK;
}

// The bf16 GEMM: the mma.sync kernel for launches of few rows, tcgen05 above
// (the same per-element arithmetic, so which one runs is work assignment).
// n_full: the output rows of the whole weight matrix that w is a row shard of
// (0: w is the whole matrix).  The accumulator sets follow from it, so the
// rows of a shard come out exactly as in the unsharded call.
// mcount (optional, device int): only rows < *mcount * mmult of x are computed.
int gemm_bf16(const void* x, int ldx, const void* w, void* y, int ldy, int y_f32, int M, int N, int K, int epi,
              int variant, void* ws, size_t ws_bytes, cudaStream_t st, const int* mcount = nullptr, int mmult = 1,
              const RopeEpi* rope = nullptr, int n_full = 0) {
  const int ks = gemm_ks(n_full > 0 ? n_full : N);
  if (M > MMA_MAX_ROWS)
    return gemm_tc(x, ldx, w, y, ldy, y_f32, M, N, K, epi, ks, variant, ws, ws_bytes, st, mcount, mmult, rope);
  const int bn = 128 / ks;
  if (N % bn)
    return set_error(BI_ERR_UNSUPPORTED, "bi_gemm: %d rows are not a multiple of the %d-row tile of the full matrix",
                     N, bn);
  int splits = 1;
  if (variant == BI_VARIANT_FAST) {
    const int kbs = gemm_kbs(bn);
    splits = gemm_fast_splits(M, (N / bn) * ((M + GEMM_BM - 1) / GEMM_BM), (K / GEMM_BK + kbs - 1) / kbs);
  }
  return gemm_mma(x, ldx, w, y, ldy, y_f32, M, N, K, epi, bn, splits, ws, ws_bytes, st, mcount, mmult, rope);
}

// w_f32: the weight is f32 (FP32-storage mode) instead of bf16.
int gemm_f32(const float* x, int ldx, const void* w, void* y, int ldy, int y_f32, int M, int N, int K, int epi,
             const int* count, cudaStream_t st, bool w_f32 = false) {
  dim3 grid((M + F32_TOK - 1) / F32_TOK, N / F32_ROWS);
  const uint16_t* wb = reinterpret_cast<const uint16_t*>(w);
  const float* wf = reinterpret_cast<const float*>(w);
  if (epi == BI_EPI_SWIGLU) {
    if (w_f32)
      BI_TRY(launch(gemm_f32_kernel<BI_EPI_SWIGLU, float>, grid, dim3(256), 0, st, x, ldx, wf, y, ldy, y_f32, M, N, K,
                    count));
    else
      BI_TRY(launch(gemm_f32_kernel<BI_EPI_SWIGLU, uint16_t>, grid, dim3(256), 0, st, x, ldx, wb, y, ldy, y_f32, M, N,
                    K, count));
  } else {
    if (w_f32)
      BI_TRY(launch(gemm_f32_kernel<BI_EPI_NONE, float>, grid, dim3(256), 0, st, x, ldx, wf, y, ldy, y_f32, M, N, K,
                    count));
    else
      BI_TRY(launch(gemm_f32_kernel<BI_EPI_NONE, uint16_t>, grid, dim3(256), 0, st, x, ldx, wb, y, ldy, y_f32, M, N, K,
                    count));
  }
  return BI_OK;
}

// ---------------------------------------------------------------- LayerCast on tensor cores
// FP32 products with bf16 weights, on the tensor cores: every f32 activation
// is split exactly into three bf16 parts x = p0 + p1 + p2 (p0 = bf16(x),
// p1 = bf16(x - p0), p2 = x - p0 - p1: 8 + 8 + 8 significant bits), every
// product of a part with a bf16 weight is exact, and each part's products are
// accumulated in fp32 over the full K in the invariant GEMM.  The three
// accumulations are added as (y0 + y1) + y2, then the epilogue runs in fp32.
// ("Give Me FP32 or Give Me Death?", LayerCast section: bf16-stored weights,
// FP32 computation.)  Per element this is independent of M, so prefill and
// decode stay bitwise equal.
__global__ void lc_split_kernel(const float* __restrict__ x, int ldx, int mb, int K, uint16_t* __restrict__ xs) {
  pdl_wait();
  pdl_trigger();
  const size_t n = (size_t)mb * K;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const size_t r = i / K, k = i % K;
    const float v = x[r * ldx + k];
    const uint16_t p0 = f32_to_bf16_bits(v);
    const float r0 = v - bf16_bits_to_f32(p0);  // exact
    const uint16_t p1 = f32_to_bf16_bits(r0);
    const float r1 = r0 - bf16_bits_to_f32(p1);  // exact, at most 8 significant bits
    xs[i] = p0;
    xs[n + i] = p1;
    xs[2 * n + i] = f32_to_bf16_bits(r1);
  }
}

__global__ void lc_combine_kernel(const float* __restrict__ yt, int mb, int N, void* __restrict__ y, int ldy,
                                  int y_f32, int swiglu) {
  pdl_wait();
  pdl_trigger();
  const int n_out = swiglu ? N / 2 : N;
  const size_t total = (size_t)mb * n_out;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total; idx += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(idx / n_out), c = (int)(idx % n_out);
    auto z = [&](int col) {
      return (yt[(size_t)r * N + col] + yt[(size_t)(mb + r) * N + col]) + yt[(size_t)(2 * mb + r) * N + col];
    };
    float v;
    if (swiglu) {
      const int blk = c / BI_GU_INTERLEAVE, rr = c % BI_GU_INTERLEAVE;
      v = silu(z(blk * 2 * BI_GU_INTERLEAVE + rr)) * z(blk * 2 * BI_GU_INTERLEAVE + BI_GU_INTERLEAVE + rr);
    } else {
      v = z(c);
    }
    store_act(y, (size_t)r * ldy + c, v, y_f32);
  }
}

// col_block > 0 (no SwiGLU epilogue): the columns in blocks of col_block
// rows of w, each block's accumulation structure fixed by the whole matrix's
// row count (n_full, else N) -- the same bits as one unblocked call.
int gemm_layercast(const float* x, int ldx, const void* w, void* y, int ldy, int y_f32, int M, int N, int K, int epi,
                   void* ws, size_t ws_bytes, cudaStream_t st, int n_full = 0, int col_block = 0) {
  const size_t need = lc_ws_bytes(M, N, K, col_block);
  BI_REQUIRE(ws && ws_bytes >= need, BI_ERR_WORKSPACE, "bi_gemm LayerCast: workspace %zu < %zu", ws_bytes, need);
  BI_REQUIRE(col_block == 0 || (col_block % 256 == 0 && epi != BI_EPI_SWIGLU), BI_ERR_INVALID_ARG,
             "LayerCast column blocks: %d", col_block);
  const int MB = std::min(M, LC_ROWS);
  const int NB = col_block > 0 ? std::min(N, col_block) : N;
  const int nf = n_full > 0 ? n_full : N;
  uint16_t* xs = reinterpret_cast<uint16_t*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
  float* yt = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(xs + (size_t)3 * MB * K) + 255) & ~uintptr_t(255));
  const size_t esz = y_f32 ? 4 : 2;
  for (int m0 = 0; m0 < M; m0 += MB) {
    const int mb = std::min(MB, M - m0);
    const size_t n = (size_t)mb * K;
    BI_TRY(launch(lc_split_kernel, dim3((int)std::min<size_t>((n + 255) / 256, 8 * (size_t)num_sms())), dim3(256), 0,
                  st, x + (size_t)m0 * ldx, ldx, mb, K, xs));
    for (int n0 = 0; n0 < N; n0 += NB) {
      const int nb = std::min(NB, N - n0);
      const int n_out = epi == BI_EPI_SWIGLU ? nb / 2 : nb;
      BI_TRY(gemm_bf16(xs, K, reinterpret_cast<const uint16_t*>(w) + (size_t)n0 * K, yt, nb, 1, 3 * mb, nb, K,
                       BI_EPI_NONE, BI_VARIANT_INVARIANT, nullptr, 0, st, nullptr, 1, nullptr, nf));
      const size_t tot = (size_t)mb * n_out;
      void* yb = reinterpret_cast<uint8_t*>(y) + ((size_t)m0 * ldy + n0) * esz;
      BI_TRY(launch(lc_combine_kernel, dim3((int)std::min<size_t>((tot + 255) / 256, 8 * (size_t)num_sms())),
                    dim3(256), 0, st, yt, mb, nb, yb, ldy, y_f32, epi == BI_EPI_SWIGLU ? 1 : 0));
    }
  }
  return BI_OK;
}

}  // namespace bi
