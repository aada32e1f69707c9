// The weight-streaming GEMM on mma.sync tensor-core tiles, for launches of
// few token rows (decode).  Per element it computes exactly what the tcgen05
// kernel computes for the same matrix (gemm_tc.cuh): the same KS interleaved
// fp32 accumulator chains in ascending K and the same fixed combining tree,
// so the two kernels give the same bits and a row's result does not depend on
// which one a launch uses.
//
// mma.sync m16n8k16 (bf16 x bf16 -> fp32) with the weight on the 16-row side
// and the tokens on the 8-column side.  Each instruction adds 16 products of
// one (n, m) pair into that pair's fp32 accumulator; the products of one
// element never meet another element's, so neither the number of token
// columns in a tile nor the tile a token lands in can change an element's
// bits.  K advances 16 at a time in ascending order; step s (k = 16s ..
// 16s+15) goes into accumulator set s % KS, and the KS sets are combined as
// ((a0 + a1) + (a2 + a3)) (KS = 4), a0 + a1 (KS = 2) or a0, where KS follows
// from the weight-row tile BN, itself chosen from N alone (gemm_ks).  The
// interleave keeps several independent mma chains per warp so the tensor-pipe
// latency is covered even when M is small.
// Weight tiles (BN rows x 64 k) and token tiles (32 rows x 64 k; only 8 or 16
// rows are copied when M is that small, since every copied row -- zero fill
// past M included -- costs the SM's copy engine the same time) stream by TMA
// (128-byte swizzle) into a multi-stage shared-memory ring filled by one
// producer warp; four consumer warps read them with ldmatrix.  The grid is
// persistent (one CTA per SM, or two with half the ring each when a launch
// has between one and two work items per SM), each CTA walking its work items
// (row group x token tile) so the ring never drains between items.
#pragma once
#include "common.cuh"
#include "gemm_tc.cuh"

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

// Work item -> (split, row group, token tile).  Splits > 1 only in the
// non-invariant FAST variant, which then writes fp32 partials per split.
template <int BN, int EPI, int MT, int CPS>
__global__ void __launch_bounds__(160, CPS)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                     void* __restrict__ y, int ldy, int y_f32, int M, int N, int K, int m_tiles, int n_groups,
                     int splits, float* __restrict__ partial, const int* __restrict__ mcount, int mmult,
                     const RopeEpi re, int xr) {
  using C = GemmCfg<BN, MT, CPS>;
  static_assert(MT == 1 || C::KS == 1, "M-blocking needs one k-phase per warp");
  static_assert(EPI != EPI_ROPE || MT == 1, "the RoPE epilogue takes one token tile per item");
  // Token rows per k-block slab of a stage: xr = 8 or 16 when M fits (MT = 1),
  // else 32.  Rows of the slab past M are zero-filled by the copy and never
  // read: the consumers stop at the last n8 tile holding live rows.
  const uint32_t stage_tx = C::W_BYTES + C::KBS * xr * MT * 128;
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
      const uint64_t wpol = l2_evict_first();  // every weight byte is read once per launch
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
            mbar_arrive_expect_tx(&full_bar[s], stage_tx);
            tma_load_3d_hint(smem + s * C::STAGE_BYTES, &tmW, 0, g * BN, (ks0 + s) * C::KBS, &full_bar[s], wpol);
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
      bool first = true, timed_out = false;
      int issued = pre;  // stages loaded so far: load n went to slot n % STAGES, phase (n / STAGES) & 1
      for (int item = blockIdx.x; item < n_items && !timed_out; item += gridDim.x) {
        int sp, g, mg;
        decode_item(item, sp, g, mg);
        const int mt = mg * MT;  // first token tile of the item
        if (mt * GEMM_BM >= Me) continue;
        const int ks0 = sp * ks_per_split;
        const int ks1 = min(kstages_total, ks0 + ks_per_split);
        for (int ks = ks0; ks < ks1; ++ks) {
          uint8_t* sb = smem + stage * C::STAGE_BYTES;
          if (!(first && ks - ks0 < pre)) {
            if (!mbar_wait(&empty_bar[stage], phase ^ 1, SITE_GEMM_EMPTY | (EPI << 12))) {
              timed_out = true;
              break;
            }
            mbar_arrive_expect_tx(&full_bar[stage], stage_tx);
            tma_load_3d_hint(sb, &tmW, 0, g * BN, ks * C::KBS, &full_bar[stage], wpol);
            ++issued;
          }
          tma_load_3d(sb + C::W_BYTES, &tmX, 0, mt * GEMM_BM, ks * C::KBS, &full_bar[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        first = false;
      }
      if (timed_out) {
        // No copy may still be writing shared memory when the CTA exits: wait
        // (bounded) for the latest load issued into each ring slot.
        for (int n = max(0, issued - C::STAGES); n < issued; ++n)
          (void)mbar_wait(&full_bar[n % C::STAGES], (uint32_t)((n / C::STAGES) & 1), SITE_GEMM_DRAIN);
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
    // RoPE epilogue (one token tile): this thread's token positions and slots,
    // and the cos/sin of its rotation pairs, requested before the K loop so
    // that the epilogue waits on no load
    int pp[4][2], ss[4][2];
    bool ok[4][2];
    if constexpr (EPI == EPI_ROPE) {
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int m = mt0 * GEMM_BM + nt * 8 + 2 * t4 + j;
          ok[nt][j] = splits == 1 && nt % C::KS == kp && nt < ntvs[0] && m < Me;
          pp[nt][j] = ok[nt][j] ? __ldg(re.pos + m) : 0;
          ss[nt][j] = ok[nt][j] ? __ldg(re.slot + m) : 0;
        }
    }
    float cs[4][2][2], sn[4][2][2];
    if constexpr (EPI == EPI_ROPE) {
      const int QD = re.Hq * re.d, KD = re.Hkv * re.d;
      const int nb = g * BN + row0;
      const bool isv = nb >= QD + KD, isq = nb < QD;
      const int rel = isq ? nb : nb - QD;
      const int e0 = (rel % re.d) >> 1;
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
            cs[nt][j][h] = ok[nt][j] ? __ldg(re.table + ti) : 0.f;
            sn[nt][j][h] = ok[nt][j] ? __ldg(re.table + ti + 1) : 0.f;
          }
        }
    }
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
        const uint32_t xb = sbase + C::W_BYTES + kb * (xr * MT * 128);
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
        // positions, slots and cos/sin of this thread's tokens came in before the K loop
        const int QD = re.Hq * re.d, KD = re.Hkv * re.d, half = re.d >> 1;
        const bool isv = nbase >= QD + KD, isq = nbase < QD;
        const int rel = isq ? nbase : nbase - QD;
        const int head = rel / re.d, e0 = (rel % re.d) >> 1;  // first-half element 16b
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
              float ra, rb;
              rope_rotate(xa, xb, cs[nt][j][h], sn[nt][j][h], ra, rb);
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

// Weight-row tile of this kernel, from N alone: 32 rows for N <= 8192 (so the
// projections of a layer spread over the SMs), else 128.
static int gemm_pick_bn(int N) {
  if (N <= 8192 && N % 32 == 0) return 32;
  if (N % 128 == 0) return 128;
  return 64;
}

// Interleaved accumulator sets of a matrix with N output rows: the four
// consumer warps of a row group take the k16 steps round-robin (4 for 32-row
// tiles, 2 for 64, 1 for 128).  A property of N, never of M; the tcgen05
// kernel reproduces it exactly.
static int gemm_ks(int N) { return 4 / (gemm_pick_bn(N) / 32); }

static int gemm_kbs(int bn, int cps = 1) {
  if (bn == 128) return cps == 2 ? GemmCfg<128, 1, 2>::KBS : GemmCfg<128>::KBS;
  return bn == 64 ? GemmCfg<64>::KBS : GemmCfg<32>::KBS;
}


template <int BN, int EPI, int MT = 1, int CPS = 1>
static int launch_gemm_bf16_t(const CUtensorMap& tw, const CUtensorMap& tx, void* y, int ldy, int y_f32, int M, int N,
                              int K, int splits, float* partial, const int* mcount, int mmult, const RopeEpi& re,
                              int xr, cudaStream_t st) {
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
                K, m_tiles, n_groups, splits, partial, mcount, mmult, re, xr));
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
// bn: the weight-row tile, 128 / KS for the matrix's KS accumulator sets.
static int gemm_mma(const void* x, int ldx, const void* w, void* y, int ldy, int y_f32, int M, int N, int K, int epi,
                    int bn, int splits, void* ws, size_t ws_bytes, cudaStream_t st, const int* mcount, int mmult,
                    const RopeEpi* rope) {
  const RopeEpi re = rope ? *rope : RopeEpi{};
  const int mt = gemm_pick_mt(bn, M);
  const int cps = gemm_pick_cps(bn, M, N, mt, splits);
  const int kbs = gemm_kbs(bn, cps);
  // token rows per copied slab: the fewest multiple of 8 (8, 16 or 32) that holds M
  const int xr = mt == 1 ? (M <= 8 ? 8 : (M <= 16 ? 16 : GEMM_BM)) : GEMM_BM;
  // 3-D views {64 k, rows, k-block}: the k-block dimension (stride 128 B) is the
  // outermost of the box, so a box lands as kbs swizzled [rows][128 B] slabs.
  CUtensorMap tw, tx;
  const uint64_t dw[3] = {(uint64_t)GEMM_BK, (uint64_t)N, (uint64_t)(K / GEMM_BK)};
  const uint64_t sw[2] = {(uint64_t)K * 2, (uint64_t)GEMM_BK * 2};
  const uint32_t bw[3] = {(uint32_t)GEMM_BK, (uint32_t)bn, (uint32_t)kbs};
  BI_TRY(encode_tmap_3d(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w, dw, sw, bw, CU_TENSOR_MAP_SWIZZLE_128B));
  const uint64_t dx[3] = {(uint64_t)GEMM_BK, (uint64_t)M, (uint64_t)(K / GEMM_BK)};
  const uint64_t sx[2] = {(uint64_t)ldx * 2, (uint64_t)GEMM_BK * 2};
  const uint32_t bx[3] = {(uint32_t)GEMM_BK, (uint32_t)(xr * mt), (uint32_t)kbs};
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
      BI_TRY((launch_gemm_bf16_t<32, EPI_ROPE, 1, 2>(tw, tx, y, ldy, y_f32, M, N, K, 1, nullptr, mcount, mmult, re, xr,
                                                    st)));
    else
      BI_TRY((launch_gemm_bf16_t<32, EPI_ROPE, 1, 1>(tw, tx, y, ldy, y_f32, M, N, K, 1, nullptr, mcount, mmult, re, xr,
                                                    st)));
    return BI_OK;
  }
#define BI_GEMM_CASE(BNV, MTV, CPSV)                                                                            \
  if (bn == BNV && mt == MTV && cps == CPSV) {                                                                  \
    if (epi == BI_EPI_SWIGLU)                                                                                   \
      BI_TRY((launch_gemm_bf16_t<BNV, BI_EPI_SWIGLU, MTV, CPSV>(tw, tx, y, ldy, y_f32, M, N, K, splits, partial,   \
                                                                mcount, mmult, re, xr, st)));                   \
    else                                                                                                        \
      BI_TRY((launch_gemm_bf16_t<BNV, BI_EPI_NONE, MTV, CPSV>(tw, tx, y, ldy, y_f32, M, N, K, splits, partial,     \
                                                              mcount, mmult, re, xr, st)));                     \
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


}  // namespace bi
