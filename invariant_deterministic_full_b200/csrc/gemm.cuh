// bi_gemm kernels.
//
// Invariance ("Meituan bitwise train/infer consistency": full-K computation in
// place of segmented reductions, one accumulation order for Prefill and
// Decode): every output element y[m][n] is accumulated in fp32 over the full K
// range, in ascending K, by the same instruction sequence whatever M is.
//
// bf16 path (gemm_bf16_kernel): mma.sync m16n8k16 (bf16 x bf16 -> fp32) with
// the weight on the 16-row side and the tokens on the 8-column side.  Each
// instruction adds 16 products of one (n, m) pair into that pair's fp32
// accumulator; the products of one element never meet another element's, so
// neither the number of token columns in a tile nor the tile a token lands in
// can change an element's bits.  K advances 16 at a time in ascending order;
// step s (k = 16s .. 16s+15) goes into accumulator set s % KS, and the KS sets
// are combined as ((a0 + a1) + (a2 + a3)) (KS = 4), a0 + a1 (KS = 2) or a0,
// where KS follows from the weight-row tile BN, itself chosen from N alone.
// The fixed interleave keeps several independent mma chains per warp so the
// tensor-pipe latency is covered even when M is small.
// Weight tiles (BN rows x 64 k) and token tiles (32 rows x 64 k) stream by TMA
// (128-byte swizzle) into a multi-stage shared-memory ring filled by one
// producer warp; four consumer warps read them with ldmatrix.  The grid is
// persistent (one CTA per SM, or two with half the ring each when a launch
// has between one and two work items per SM), each CTA walking its work items
// (row group x token tile) so the ring never drains between items.
//
// LayerCast ("Give Me FP32 or Give Me Death?", LayerCast section: bf16-stored
// weights, fp32 arithmetic) has two routes.  Projections (gemm_layercast, at
// the end of this file) split each f32 activation exactly into three bf16
// parts and run them through gemm_bf16_kernel.  The LM head
// (gemm_f32_kernel) upcasts the weight from bf16 to fp32 in registers and
// takes every product and sum as an fp32 FMA.  Element order there: lane l of
// a warp owns the k-slices [256 i + 8 l, 256 i + 8 l + 8) for i = 0, 1, ...;
// it accumulates them with sequential FMAs in ascending k, and the 32 lane
// partials are then combined by a fixed xor-butterfly.  This is the same for
// every M and every row/token tiling.
#pragma once
#include "common.cuh"

namespace bi {

constexpr int GEMM_BM = 32;  // token rows per tile (fixed; never depends on M)
constexpr int GEMM_BK = 64;  // k per k-block (128 bytes of bf16: one swizzled smem line)

// One ring stage holds KBS consecutive k-blocks of the weight tile (BN rows)
// and of the token tile (32 rows), each fetched by ONE 3-D TMA operation whose
// box is {64 k, rows, KBS k-blocks}: the k-block dimension is the outermost of
// the box, so in shared memory every k-block is a [rows][128 B] slab with the
// 128-byte swizzle -- the layout ldmatrix reads without bank conflicts.  Few,
// large TMA operations per stage keep each SM streaming near its peak rate.
//
// Consumer warps: RW = BN/32 row groups x KS k-phases.  Warp (rw, kp) owns the
// weight rows [32 rw, 32 rw + 32) and all 32 token columns, and takes the k16
// steps whose index within their 64-k block is congruent to kp modulo KS: its
// accumulators are the KS-interleaved accumulator set kp of those outputs.
// Every weight and token fragment is therefore read from shared memory once
// per row group, and the sets meet in a fixed tree after the K loop.
// MT: 32-row token tiles sharing each weight stage (M-blocking; a property of
// the launch, not of the arithmetic: every element still sees the same
// instruction sequence).  MT > 1 only with 128-row weight tiles.
// CPS: CTAs per SM.  1: one persistent CTA per SM with a ~212 KB ring.  2:
// two CTAs of ~112 KB each, for launches with between 1x and 2x as many work
// items as SMs -- an SM that holds two row groups then streams both at once
// instead of one after the other, so the extra groups do not double its time.
template <int BN, int MT = 1, int CPS = 1>
struct GemmCfg {
  static constexpr int KBS = BN == 128 ? (CPS == 2 ? 1 : 2) : 4;
  static constexpr int W_BYTES = KBS * BN * 128;
  static constexpr int X_BYTES = KBS * GEMM_BM * MT * 128;
  static constexpr int STAGE_BYTES = W_BYTES + X_BYTES;
  static constexpr int RW = BN / 32;      // row groups (32 weight rows each)
  // Interleaved accumulator sets per output element (a property of the matrix
  // shape through BN, never of M), one per k-phase warp of a row group.
  static constexpr int KS = 4 / RW;
  // cross-warp partial sums: each warp parks the 8 values x 32 lanes of every
  // n8 token tile that another warp of its row group finishes
  static constexpr int RED_TILES = KS > 1 ? 4 - 4 / KS : 0;
  static constexpr int RED_BYTES = 4 * RED_TILES * 8 * 32 * 4;
  static constexpr int STAGES = ((CPS == 2 ? 112 : 212) * 1024 - RED_BYTES) / STAGE_BYTES;
  static constexpr int SMEM = STAGES * STAGE_BYTES + RED_BYTES + 1024;
};

// Fused RoPE + KV-append epilogue of the QKV projection (bf16 mode).  The
// fused QKV weight stores each q/k head in the "paired" row order: in every
// 32-row block b of a head, rows 0..15 are elements 16b..16b+15 and rows
// 16..31 their rotate-half partners d/2 + 16b .. d/2 + 16b + 15 (v rows keep
// their natural order).  A warp's two 16-row tiles then hold both members of
// each rotation pair for its tokens, so the epilogue rotates in registers
// (x' = x c - y s, y' = y c + x s, (c, s) from the f32 table at the token's
// position), writes q in the activation dtype and appends k and v to the cache.
constexpr int EPI_ROPE = 2;
struct RopeEpi {
  const float* table;
  int table_max_pos;
  void* q_out;
  void* kc;
  void* vc;
  const int32_t* slot;
  const int32_t* pos;
  int Hq, Hkv, d, layer, n_layers, n_slots, cap;
};

// Work item -> (split, row group, token tile).  Splits > 1 only in the
// non-invariant FAST variant, which then writes fp32 partials per split.
template <int BN, int EPI, int MT, int CPS>
__global__ void __launch_bounds__(160, CPS)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                     void* __restrict__ y, int ldy, int y_f32, int M, int N, int K, int m_tiles, int n_groups,
                     int splits, float* __restrict__ partial, const int* __restrict__ mcount, int mmult,
                     const RopeEpi re) {
  using C = GemmCfg<BN, MT, CPS>;
  static_assert(MT == 1 || C::KS == 1, "M-blocking needs one k-phase per warp");
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[C::STAGES];
  __shared__ __align__(8) uint64_t empty_bar[C::STAGES];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // stages of KBS k-blocks; a final partial stage reads zeros past K (TMA fill),
  // which add exact zeros to the accumulators
  const int kstages_total = (K / GEMM_BK + C::KBS - 1) / C::KBS;
  const int ks_per_split = (kstages_total + splits - 1) / splits;
  const int m_groups = (m_tiles + MT - 1) / MT;  // MT token tiles per work item
  const int n_items = splits * n_groups * m_groups;
  // Work item -> (split, weight row group, token group).  Token group fastest by
  // default (CTAs working at the same time share weight tiles in L2); with a
  // device-side row count, token group slowest, so the live first token tiles
  // are spread over all CTAs.
  const bool mg_major = mcount != nullptr;
  auto decode_item = [&](int item, int& sp, int& g, int& mg) {
    if (mg_major) {
      g = item % n_groups;
      sp = (item / n_groups) % splits;
      mg = item / (n_groups * splits);
    } else {
      mg = item % m_groups;
      g = (item / m_groups) % n_groups;
      sp = item / (m_groups * n_groups);
    }
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 4);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 4) {  // ---------------- producer: one elected lane issues TMA
    if (lane == 0) {
      prefetch_tmap(&tmW);
      prefetch_tmap(&tmX);
      // Prologue: the first ring stages of weight tiles depend on no earlier
      // kernel, so they are requested before waiting for the previous launch.
      // (With a device-side row count only token group 0 is sure to be live:
      // it is live unless the count is zero, and then the prefetched stages
      // are drained before the CTA exits.)
      int pre = 0;
      if ((int)blockIdx.x < n_items) {
        int sp, g, mg;
        decode_item(blockIdx.x, sp, g, mg);
        if (mcount == nullptr || mg == 0) {
          const int ks0 = sp * ks_per_split;
          const int ks1 = min(kstages_total, ks0 + ks_per_split);
          pre = max(0, min(C::STAGES, ks1 - ks0));
          for (int s = 0; s < pre; ++s) {
            mbar_arrive_expect_tx(&full_bar[s], C::STAGE_BYTES);
            tma_load_3d(smem + s * C::STAGE_BYTES, &tmW, 0, g * BN, (ks0 + s) * C::KBS, &full_bar[s]);
          }
        }
      }
      pdl_wait();
      pdl_trigger();
      // rows beyond a device-side count (selective recompute) are not computed
      const int Me = mcount ? min(M, *mcount * mmult) : M;
      if (pre > 0 && Me <= 0) {
        // Nothing to compute.  Each prefetched stage's barrier also expects its
        // token tile: load those (row 0 on, in bounds or zero-filled) so the
        // barriers complete, wait for them, then leave.
        int sp, g, mg;
        decode_item(blockIdx.x, sp, g, mg);
        for (int s = 0; s < pre; ++s)
          tma_load_3d(smem + s * C::STAGE_BYTES + C::W_BYTES, &tmX, 0, 0, (sp * ks_per_split + s) * C::KBS,
                      &full_bar[s]);
        for (int s = 0; s < pre; ++s) (void)mbar_wait(&full_bar[s], 0u, SITE_GEMM_DRAIN);
        return;
      }
      int stage = 0;
      uint32_t phase = 0;
      bool first = true;
      for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        int sp, g, mg;
        decode_item(item, sp, g, mg);
        const int mt = mg * MT;  // first token tile of the item
        if (mt * GEMM_BM >= Me) continue;
        const int ks0 = sp * ks_per_split;
        const int ks1 = min(kstages_total, ks0 + ks_per_split);
        for (int ks = ks0; ks < ks1; ++ks) {
          uint8_t* sb = smem + stage * C::STAGE_BYTES;
          if (!(first && ks - ks0 < pre)) {
            if (!mbar_wait(&empty_bar[stage], phase ^ 1, SITE_GEMM_EMPTY | (EPI << 12))) return;
            mbar_arrive_expect_tx(&full_bar[stage], C::STAGE_BYTES);
            tma_load_3d(sb, &tmW, 0, g * BN, ks * C::KBS, &full_bar[stage]);
          }
          tma_load_3d(sb + C::W_BYTES, &tmX, 0, mt * GEMM_BM, ks * C::KBS, &full_bar[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        first = false;
      }
    }
    return;
  }
  pdl_wait();
  pdl_trigger();

  // ---------------- consumers
  const int rw = warp % C::RW, kp = warp / C::RW;
  const int row0 = rw * 32;                      // weight rows [row0, row0+32) of the tile
  const int g8 = lane >> 2, t4 = lane & 3;
  float* red = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES);  // [warp][32 values][32 lanes]
  int stage = 0;
  uint32_t phase = 0;
  // A ring wait that runs out (error flag set) stops this warp's waits and
  // math, but it keeps meeting the named barriers so no warp waits forever.
  bool dead = false;
  const int Me = mcount ? min(M, *mcount * mmult) : M;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    int sp, g, mg;
    decode_item(item, sp, g, mg);
    const int mt0 = mg * MT;
    if (mt0 * GEMM_BM >= Me) continue;
    const int ks0 = sp * ks_per_split;
    const int ks1 = min(kstages_total, ks0 + ks_per_split);
    int ntvs[MT];  // n8 token tiles holding live rows, per token tile
#pragma unroll
    for (int j = 0; j < MT; ++j) ntvs[j] = max(0, min(4, (Me - (mt0 + j) * GEMM_BM + 7) / 8));
    // accumulator set kp of this warp's outputs: k16 steps kk = kp, kp + KS, ... of every 64-k block
    float accm[MT][2][4][4];
#pragma unroll
    for (int j = 0; j < MT; ++j)
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
          for (int c = 0; c < 4; ++c) accm[j][a][b][c] = 0.f;

    for (int ks = ks0; ks < ks1; ++ks) {
      if (!dead && !mbar_wait(&full_bar[stage], phase, SITE_GEMM_FULL | (EPI << 12))) dead = true;
      const uint32_t sbase = smem_u32(smem + stage * C::STAGE_BYTES);
#pragma unroll
      for (int kb = 0; kb < C::KBS && !dead; ++kb) {
        const uint32_t wb = sbase + kb * (BN * 128);
        const uint32_t xb = sbase + C::W_BYTES + kb * (GEMM_BM * MT * 128);
#pragma unroll
        for (int j = 0; j < 4 / C::KS; ++j) {
          const int kk = kp + j * C::KS;
          uint32_t a[2][4];
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int row = row0 + r * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
            ldsm_x4(swz128(wb, row, 2 * kk + (lane >> 4)), a[r][0], a[r][1], a[r][2], a[r][3]);
          }
#pragma unroll
          for (int j = 0; j < MT; ++j) {
            const int ntv = ntvs[j];
            uint32_t b[4][2];
#pragma unroll
            for (int p = 0; p < 2; ++p) {
              if (2 * p < ntv) {
                const int tok = j * GEMM_BM + p * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
                ldsm_x4(swz128(xb, tok, 2 * kk + ((lane >> 3) & 1)), b[2 * p][0], b[2 * p][1], b[2 * p + 1][0],
                        b[2 * p + 1][1]);
              }
            }
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
              for (int nt = 0; nt < 4; ++nt)
                if (nt < ntv) mma_bf16_16816(accm[j][r][nt], a[r], b[nt][0], b[nt][1]);
          }
        }
      }
      __syncwarp();
      if (lane == 0 && !dead) mbar_arrive(&empty_bar[stage]);
      if (++stage == C::STAGES) {
        stage = 0;
        phase ^= 1;
      }
    }
#pragma unroll
    for (int jt = 0; jt < MT; ++jt) {
    const int mt = mt0 + jt;
    const int ntv = ntvs[jt];
    float (&acc)[2][4][4] = accm[jt];
    if (ntv == 0) continue;  // uniform across the consumer warps
    if constexpr (C::KS > 1) {
      // The KS sets of the row group meet through shared memory: warp (rw, kp)
      // finishes the n8 token tiles nt = kp, kp + KS, ... combining
      // ((s0 + s1) + (s2 + s3)) (KS = 4) or s0 + s1 (KS = 2), set j coming from
      // warp (rw, j); the epilogue work is shared by all four warps.
      // slot of tile b among the RED_TILES tiles that warp (rw, j) parks: the tiles it
      // does not finish, in ascending order
      auto slot = [&](int b, int j) { return b / C::KS * (C::KS - 1) + (b % C::KS) - (b % C::KS > j ? 1 : 0); };
      auto cell = [&](int w, int sl, int a, int c) { return ((w * C::RED_TILES + sl) * 8 + a * 4 + c) * 32 + lane; };
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        if (b % C::KS == kp) continue;
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int c = 0; c < 4; ++c) red[cell(warp, slot(b, kp), a, c)] = acc[a][b][c];
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        if (b % C::KS != kp) continue;
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float sv[4];
#pragma unroll
            for (int j = 0; j < C::KS; ++j)
              sv[j] = j == kp ? acc[a][b][c] : red[cell(rw + C::RW * j, slot(b, j), a, c)];
            if constexpr (C::KS == 4)
              acc[a][b][c] = (sv[0] + sv[1]) + (sv[2] + sv[3]);
            else
              acc[a][b][c] = sv[0] + sv[1];
          }
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");  // the next item reuses the exchange buffer
    }
    if (dead) continue;

    // ---------------- epilogue: fragment (row g8 (+8), cols 2*t4 (+1)) of each m16n8 tile
    const int nbase = g * BN + row0;
    if constexpr (EPI == EPI_ROPE) {
      if (splits == 1) {
        // positions, slots and cos/sin of this thread's tokens are all fetched
        // before any store, so the dependent loads overlap
        const int QD = re.Hq * re.d, KD = re.Hkv * re.d, half = re.d >> 1;
        const bool isv = nbase >= QD + KD, isq = nbase < QD;
        const int rel = isq ? nbase : nbase - QD;
        const int head = rel / re.d, e0 = (rel % re.d) >> 1;  // first-half element 16b
        int pp[4][2], ss[4][2];
        bool ok[4][2];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int m = mt * GEMM_BM + nt * 8 + 2 * t4 + j;
            ok[nt][j] = nt % C::KS == kp && nt < ntv && m < Me;
            pp[nt][j] = ok[nt][j] ? __ldg(re.pos + m) : 0;
            ss[nt][j] = ok[nt][j] ? __ldg(re.slot + m) : 0;
          }
        float cs[4][2][2], sn[4][2][2];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int p = pp[nt][j], sl = ss[nt][j];
            if (ok[nt][j] && (p < 0 || p >= re.cap || p >= re.table_max_pos || sl < 0 || sl >= re.n_slots)) {
              dev_flag(DEVERR_CAPACITY);
              ok[nt][j] = false;
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const size_t ti = (size_t)(ok[nt][j] && !isv ? p : 0) * re.d + 2 * (e0 + g8 + h * 8);
              cs[nt][j][h] = __ldg(re.table + ti);
              sn[nt][j][h] = __ldg(re.table + ti + 1);
            }
          }
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int j = i & 1, h = i >> 1;
            if (!ok[nt][j]) continue;
            const int m = mt * GEMM_BM + nt * 8 + 2 * t4 + j;
            const int p = pp[nt][j], sl = ss[nt][j];
            const int rin = g8 + h * 8;
            if (!isv) {
              const int ei = e0 + rin;
              const float xa = acc[0][nt][i], xb = acc[1][nt][i];
              const float ra = xa * cs[nt][j][h] - xb * sn[nt][j][h];
              const float rb = xb * cs[nt][j][h] + xa * sn[nt][j][h];
              if (isq) {
                store_act(re.q_out, (size_t)m * QD + head * re.d + ei, ra, false);
                store_act(re.q_out, (size_t)m * QD + head * re.d + ei + half, rb, false);
              } else {
                const size_t crow = (((size_t)sl * re.n_layers + re.layer) * re.Hkv + head) * re.cap + p;
                store_act(re.kc, crow * re.d + ei, ra, false);
                store_act(re.kc, crow * re.d + ei + half, rb, false);
              }
            } else {
#pragma unroll
              for (int r = 0; r < 2; ++r) {
                const int ev = nbase - QD - KD + r * 16 + rin;
                const size_t crow = (((size_t)sl * re.n_layers + re.layer) * re.Hkv + ev / re.d) * re.cap + p;
                store_act(re.vc, crow * re.d + ev % re.d, acc[r][nt][i], false);
              }
            }
          }
        continue;
      }
    }
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      if (nt >= ntv || nt % C::KS != kp) continue;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = mt * GEMM_BM + nt * 8 + 2 * t4 + (i & 1);
        if (m >= Me) continue;
        const int rin = g8 + (i >> 1) * 8;
        if (splits > 1) {  // FAST variant: raw fp32 partial of this split
#pragma unroll
          for (int r = 0; r < 2; ++r)
            partial[((size_t)sp * M + m) * N + nbase + r * 16 + rin] = acc[r][nt][i];
        } else if constexpr (EPI == BI_EPI_SWIGLU) {
          const int col = (nbase >> 1) + rin;  // 32-row block -> 16 output columns
          store_act(y, (size_t)m * ldy + col, silu(acc[0][nt][i]) * acc[1][nt][i], y_f32);
        } else {
#pragma unroll
          for (int r = 0; r < 2; ++r) store_act(y, (size_t)m * ldy + nbase + r * 16 + rin, acc[r][nt][i], y_f32);
        }
      }
    }
    }  // token tiles of the item
  }
}

// FAST variant: y = sum over splits (ascending) of the fp32 partials, then the epilogue.
template <int EPI>
__global__ void splitk_reduce_kernel(const float* __restrict__ partial, void* __restrict__ y, int ldy, int y_f32, int M,
                                     int N, int splits) {
  pdl_wait();
  pdl_trigger();
  const int n_out = EPI == BI_EPI_SWIGLU ? N / 2 : N;
  const size_t total = (size_t)M * n_out;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total; idx += (size_t)gridDim.x * blockDim.x) {
    const int m = (int)(idx / n_out), c = (int)(idx % n_out);
    if constexpr (EPI == BI_EPI_SWIGLU) {
      const int blk = c / 16, r = c % 16;
      const int ng = blk * 32 + r, nu = ng + 16;
      float sg = 0.f, su = 0.f;
      for (int s = 0; s < splits; ++s) {
        sg += partial[((size_t)s * M + m) * N + ng];
        su += partial[((size_t)s * M + m) * N + nu];
      }
      store_act(y, (size_t)m * ldy + c, silu(sg) * su, y_f32);
    } else {
      float s0 = 0.f;
      for (int s = 0; s < splits; ++s) s0 += partial[((size_t)s * M + m) * N + c];
      store_act(y, (size_t)m * ldy + c, s0, y_f32);
    }
  }
}

// ---------------------------------------------------------------- LayerCast (fp32 FMA)
constexpr int F32_ROWS = 32;  // weight rows per CTA (8 warps x 4 rows)
constexpr int F32_TOK = 16;   // token columns per CTA
constexpr int F32_KC = 256;   // k per chunk (32 lanes x 8)

// x: f32 [M][ldx]; w: bf16 [N][K]; y: [M][ldy].  Optional device row count
// (count != nullptr): only token rows < *count are computed (used by the
// selective recompute, whose row count is known only on the device).
// The CTA's 16 token rows are staged chunk by chunk (256 k) in shared memory,
// double-buffered, and read by all 8 warps; each warp streams 4 weight rows.
template <int EPI>
__global__ void __launch_bounds__(256)
    gemm_f32_kernel(const float* __restrict__ x, int ldx, const uint16_t* __restrict__ w, void* __restrict__ y,
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
      uint4 u[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) u[r] = __ldg(reinterpret_cast<const uint4*>(w + (size_t)rows[r] * K + k));
#pragma unroll
      for (int t = 0; t < F32_TOK; ++t) {
        if (t < ntok) {
          const float4 x0 = *reinterpret_cast<const float4*>(&xs[buf][t][8 * lane]);
          const float4 x1 = *reinterpret_cast<const float4*>(&xs[buf][t][8 * lane + 4]);
          const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              const uint32_t word = j < 2 ? u[r].x : j < 4 ? u[r].y : j < 6 ? u[r].z : u[r].w;
              const float wv = (j & 1) ? bf16hi(word) : bf16lo(word);
              acc[r][t] = fmaf(wv, xv[j], acc[r][t]);
            }
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
static int gemm_pick_bn(int N) {
  if (N <= 8192 && N % 32 == 0) return 32;
  if (N % 128 == 0) return 128;
  return 64;
}

// Split factor of the FAST variant: more K splits for small M so that the
// grid fills the SMs (the usual library heuristic) -- which is exactly what
// makes the result depend on the batch size.
static int gemm_kbs(int bn, int cps = 1) {
  if (bn == 128) return cps == 2 ? GemmCfg<128, 1, 2>::KBS : GemmCfg<128>::KBS;
  return bn == 64 ? GemmCfg<64>::KBS : GemmCfg<32>::KBS;
}

static int gemm_fast_splits(int M, int n_items, int kstages) {
  const int sms = num_sms();
  if (M > 16) return 1;
  int s = (2 * sms + n_items - 1) / n_items;
  if (M <= 4) s *= 2;
  s = s < 1 ? 1 : (s > 8 ? 8 : s);
  while (s > 1 && kstages / s < 2) --s;
  return s;
}

// LayerCast on tensor cores: rows of x per pass (bounds the workspace)
constexpr int LC_ROWS = 256;
static size_t lc_ws_bytes(int M, int N, int K) {
  const size_t mb = (size_t)std::min(M, LC_ROWS);
  return 3 * mb * K * 2 + 3 * mb * N * 4 + 512;
}

size_t gemm_ws_bytes(int M, int N, int K, int mode, int variant) {
  if (mode == BI_MODE_LAYERCAST) return M > 0 ? lc_ws_bytes(M, N, K) : 0;
  if (variant != BI_VARIANT_FAST) return 0;
  const int bn = gemm_pick_bn(N);
  const int items = (N / bn) * ((M + GEMM_BM - 1) / GEMM_BM);
  const int kbs = gemm_kbs(bn);
  const int s = gemm_fast_splits(M, items, (K / GEMM_BK + kbs - 1) / kbs);
  return s > 1 ? (size_t)s * M * N * sizeof(float) : 0;
}

template <int BN, int EPI, int MT = 1, int CPS = 1>
static int launch_gemm_bf16_t(const CUtensorMap& tw, const CUtensorMap& tx, void* y, int ldy, int y_f32, int M, int N,
                              int K, int splits, float* partial, const int* mcount, int mmult, const RopeEpi& re,
                              cudaStream_t st) {
  using C = GemmCfg<BN, MT, CPS>;
  static bool attr_done = false;  // per instantiation; set once per process
  if (!attr_done) {
    BI_CHECK_CUDA(cudaFuncSetAttribute(gemm_bf16_kernel<BN, EPI, MT, CPS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
    attr_done = true;
  }
  const int m_tiles = (M + GEMM_BM - 1) / GEMM_BM;
  const int n_groups = N / BN;
  const int items = splits * n_groups * ((m_tiles + MT - 1) / MT);
  const int grid = items < CPS * num_sms() ? items : CPS * num_sms();
  BI_TRY(launch(gemm_bf16_kernel<BN, EPI, MT, CPS>, dim3(grid), dim3(160), C::SMEM, st, tw, tx, y, ldy, y_f32, M, N,
                K, m_tiles, n_groups, splits, partial, mcount, mmult, re));
  return BI_OK;
}

// Two CTAs per SM when the launch has between 1x and 2x as many work items as
// SMs (one token tile per item, no split).
static int gemm_pick_cps(int bn, int M, int N, int mt, int splits) {
  if (mt != 1 || splits != 1) return 1;
  const int items = (N / bn) * ((M + GEMM_BM - 1) / GEMM_BM);
  return items > num_sms() && items <= 2 * num_sms() ? 2 : 1;
}

// Token tiles per weight stage: 4 for 128-row weight tiles once M spans four
// token tiles (prefill: the weight is then read once per 128 token rows), else 1.
static int gemm_pick_mt(int bn, int M) { return bn == 128 && M >= 4 * GEMM_BM ? 4 : 1; }

// mcount (optional, device int): only rows < *mcount * mmult of x are computed.
int gemm_bf16(const void* x, int ldx, const void* w, void* y, int ldy, int y_f32, int M, int N, int K, int epi,
              int variant, void* ws, size_t ws_bytes, cudaStream_t st, const int* mcount = nullptr, int mmult = 1,
              const RopeEpi* rope = nullptr) {
  const RopeEpi re = rope ? *rope : RopeEpi{};
  const int bn = gemm_pick_bn(N);
  const int mt = gemm_pick_mt(bn, M);
  int splits = 1;
  if (variant == BI_VARIANT_FAST) {
    const int items = (N / bn) * ((M + GEMM_BM - 1) / GEMM_BM);
    const int kbs1 = gemm_kbs(bn);
    splits = gemm_fast_splits(M, items, (K / GEMM_BK + kbs1 - 1) / kbs1);
  }
  const int cps = gemm_pick_cps(bn, M, N, mt, splits);
  const int kbs = gemm_kbs(bn, cps);
  // 3-D views {64 k, rows, k-block}: the k-block dimension (stride 128 B) is the
  // outermost of the box, so a box lands as kbs swizzled [rows][128 B] slabs.
  CUtensorMap tw, tx;
  const uint64_t dw[3] = {(uint64_t)GEMM_BK, (uint64_t)N, (uint64_t)(K / GEMM_BK)};
  const uint64_t sw[2] = {(uint64_t)K * 2, (uint64_t)GEMM_BK * 2};
  const uint32_t bw[3] = {(uint32_t)GEMM_BK, (uint32_t)bn, (uint32_t)kbs};
  BI_TRY(encode_tmap_3d(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w, dw, sw, bw, CU_TENSOR_MAP_SWIZZLE_128B));
  const uint64_t dx[3] = {(uint64_t)GEMM_BK, (uint64_t)M, (uint64_t)(K / GEMM_BK)};
  const uint64_t sx[2] = {(uint64_t)ldx * 2, (uint64_t)GEMM_BK * 2};
  const uint32_t bx[3] = {(uint32_t)GEMM_BK, (uint32_t)(GEMM_BM * mt), (uint32_t)kbs};
  BI_TRY(encode_tmap_3d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, dx, sx, bx, CU_TENSOR_MAP_SWIZZLE_128B));
  float* partial = nullptr;
  if (splits > 1) {
    const size_t need = (size_t)splits * M * N * sizeof(float);
    BI_REQUIRE(ws && ws_bytes >= need, BI_ERR_WORKSPACE, "bi_gemm FAST: workspace %zu < %zu", ws_bytes, need);
    partial = reinterpret_cast<float*>(ws);
  }
  if (epi == EPI_ROPE) {
    if (bn != 32 || splits > 1 || !rope)
      return set_error(BI_ERR_UNSUPPORTED, "fused RoPE epilogue needs the 32-row tile and no split");
    if (cps == 2)
      BI_TRY((launch_gemm_bf16_t<32, EPI_ROPE, 1, 2>(tw, tx, y, ldy, y_f32, M, N, K, 1, nullptr, mcount, mmult, re, st)));
    else
      BI_TRY((launch_gemm_bf16_t<32, EPI_ROPE, 1, 1>(tw, tx, y, ldy, y_f32, M, N, K, 1, nullptr, mcount, mmult, re, st)));
    return BI_OK;
  }
#define BI_GEMM_CASE(BNV, MTV, CPSV)                                                                            \
  if (bn == BNV && mt == MTV && cps == CPSV) {                                                                  \
    if (epi == BI_EPI_SWIGLU)                                                                                   \
      BI_TRY((launch_gemm_bf16_t<BNV, BI_EPI_SWIGLU, MTV, CPSV>(tw, tx, y, ldy, y_f32, M, N, K, splits, partial,   \
                                                                mcount, mmult, re, st)));                       \
    else                                                                                                        \
      BI_TRY((launch_gemm_bf16_t<BNV, BI_EPI_NONE, MTV, CPSV>(tw, tx, y, ldy, y_f32, M, N, K, splits, partial,     \
                                                              mcount, mmult, re, st)));                         \
  }
  BI_GEMM_CASE(32, 1, 1)
  BI_GEMM_CASE(64, 1, 1)
  BI_GEMM_CASE(128, 1, 1)
  BI_GEMM_CASE(128, 4, 1)
  BI_GEMM_CASE(32, 1, 2)
  BI_GEMM_CASE(64, 1, 2)
  BI_GEMM_CASE(128, 1, 2)
#undef BI_GEMM_CASE
  if (splits > 1) {
    const int n_out = epi == BI_EPI_SWIGLU ? N / 2 : N;
    const size_t total = (size_t)M * n_out;
    int blocks = (int)((total + 255) / 256);
    if (blocks > 4 * num_sms()) blocks = 4 * num_sms();
    if (epi == BI_EPI_SWIGLU)
      BI_TRY(launch(splitk_reduce_kernel<BI_EPI_SWIGLU>, dim3(blocks), dim3(256), 0, st, partial, y, ldy, y_f32, M, N, splits));
    else
      BI_TRY(launch(splitk_reduce_kernel<BI_EPI_NONE>, dim3(blocks), dim3(256), 0, st, partial, y, ldy, y_f32, M, N, splits));
  }
  return BI_OK;
}

int gemm_f32(const float* x, int ldx, const void* w, void* y, int ldy, int y_f32, int M, int N, int K, int epi,
             const int* count, cudaStream_t st) {
  dim3 grid((M + F32_TOK - 1) / F32_TOK, N / F32_ROWS);
  if (epi == BI_EPI_SWIGLU)
    BI_TRY(launch(gemm_f32_kernel<BI_EPI_SWIGLU>, dim3(grid), dim3(256), 0, st, x, ldx, reinterpret_cast<const uint16_t*>(w), y, ldy, y_f32,
                                                         M, N, K, count));
  else
    BI_TRY(launch(gemm_f32_kernel<BI_EPI_NONE>, dim3(grid), dim3(256), 0, st, x, ldx, reinterpret_cast<const uint16_t*>(w), y, ldy, y_f32, M,
                                                       N, K, count));
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

int gemm_layercast(const float* x, int ldx, const void* w, void* y, int ldy, int y_f32, int M, int N, int K, int epi,
                   void* ws, size_t ws_bytes, cudaStream_t st) {
  const size_t need = lc_ws_bytes(M, N, K);
  BI_REQUIRE(ws && ws_bytes >= need, BI_ERR_WORKSPACE, "bi_gemm LayerCast: workspace %zu < %zu", ws_bytes, need);
  const int MB = std::min(M, LC_ROWS);
  uint16_t* xs = reinterpret_cast<uint16_t*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
  float* yt = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(xs + (size_t)3 * MB * K) + 255) & ~uintptr_t(255));
  const int n_out = epi == BI_EPI_SWIGLU ? N / 2 : N;
  for (int m0 = 0; m0 < M; m0 += MB) {
    const int mb = std::min(MB, M - m0);
    const size_t n = (size_t)mb * K;
    BI_TRY(launch(lc_split_kernel, dim3((int)std::min<size_t>((n + 255) / 256, 8 * (size_t)num_sms())), dim3(256), 0,
                  st, x + (size_t)m0 * ldx, ldx, mb, K, xs));
    BI_TRY(gemm_bf16(xs, K, w, yt, N, 1, 3 * mb, N, K, BI_EPI_NONE, BI_VARIANT_INVARIANT, nullptr, 0, st));
    const size_t tot = (size_t)mb * n_out;
    void* yb = reinterpret_cast<uint8_t*>(y) + (size_t)m0 * ldy * (y_f32 ? 4 : 2);
    BI_TRY(launch(lc_combine_kernel, dim3((int)std::min<size_t>((tot + 255) / 256, 8 * (size_t)num_sms())), dim3(256),
                  0, st, yt, mb, N, yb, ldy, y_f32, epi == BI_EPI_SWIGLU ? 1 : 0));
  }
  return BI_OK;
}

}  // namespace bi
