// bi_gemm on the 5th-generation tensor cores (tcgen05 + TMEM), bf16 x bf16 -> fp32.
//
// Invariance ("Meituan bitwise train/infer consistency": full-K computation in
// place of segmented reductions, one accumulation order for Prefill and
// Decode).  Every output element y[m][n] is the fixed combination of KS fp32
// accumulators in TMEM: set j is a chain of tcgen05.mma.kind::f16 instructions
// of shape M = 128 (token rows) x N (weight rows) x K = 16 over the k16 steps
// s = j, j + KS, ... in ascending order (the first with the accumulator
// disabled), and the sets meet as ((s0 + s1) + (s2 + s3)), s0 + s1 or s0.  KS
// is a property of the matrix (gemm_ks: from N alone), the same as in the
// mma.sync kernel used for few-row launches (gemm_mma.cuh).  Each instruction
// adds the 16 products of row m of the token operand and row n of the weight
// operand to that element's accumulator; an element's result depends only on
// its own two rows.  So which 128-row token tile a token lands in, how many
// live tokens the tile holds, how many token tiles share a weight stage, and
// the instruction's N (the weight tile, chosen per launch) change no bits.
// The instruction-shape check confirmed this on B200 -- the same elements
// through N = 32 .. 256, with rows permuted, with the other rows replaced by
// garbage, and against an mma.sync m16n8k16 chain over the same k-slices, all
// bit-identical -- and the invariance tests guard it end to end.
//
// Data flow per CTA (persistent, 192 threads):
//   warp 4      producer: one lane issues TMA loads of the weight tile
//               (BN rows x 64 k per k-block, 128-byte swizzle) and the token
//               tile(s) into a ring of shared-memory stages; the first stages
//               of weights are requested before the programmatic-dependency
//               wait (they depend on no earlier kernel);
//   warp 5      MMA issuer: allocates TMEM, one lane issues the MMAs of each
//               stage and releases the stage with tcgen05.commit; a commit
//               after an item's last stage hands the accumulator to the
//               epilogue (double-buffered when TMEM allows);
//   warps 0..3  epilogue: warp w reads TMEM lanes 32w..32w+31 (one token row
//               per thread, 32 columns at a time), applies the epilogue
//               (none / SwiGLU / RoPE + KV append / split-K partial) and stores.
// Decode tiles stage only the 32 live token rows: the MMA's rows 32..127 then
// read whatever follows in shared memory (other slabs of the ring), which only
// reaches accumulator rows that are never stored.
//
// Every wait is bounded (1 s); a wait that runs out flags the device error
// word and marks the CTA dead: the other roles skip their remaining waits, the
// producer waits (bounded) for its outstanding copies, the MMA lane waits for
// its outstanding MMAs, and TMEM is freed before the CTA exits.
#pragma once
#include "common.cuh"

namespace bi {

// ---------------------------------------------------------------- tcgen05 primitives
// Shared-memory matrix descriptor, K-major operand written by TMA with the
// 128-byte swizzle: 8-row groups 1024 bytes apart (stride byte offset), the
// leading byte offset unused for swizzled K-major layouts (1), descriptor
// version 1, swizzle mode 2 (128 B).
__device__ __forceinline__ uint64_t umma_sdesc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
// Arrive once on `bar` when every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// 32 TMEM lanes (thread t of the warp: lane base + t) x 32 columns of 32 bits.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

constexpr int TC_THREADS = 192;  // 4 epilogue warps, producer warp, MMA warp
constexpr int TC_TILE_M = 128;   // token rows per MMA (fixed instruction M)
constexpr int TC_BK = 64;        // k per k-block: one 128-byte swizzled row of bf16

// BN: weight rows per item (the MMA's N); MT: 128-row token tiles per item
// (each its own accumulator; prefill M-blocking); XR: token rows staged per
// tile (32 for launches of at most 32 rows, else 128); KS: interleaved
// accumulator sets (k16 step s goes to set s % KS; a property of the matrix,
// see gemm_ks); CPS: CTAs per SM.
template <int BN, int MT, int XR, int KS, int CPS>
struct TcCfg {
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "weight tile");
  static_assert(XR == 32 || XR == 128, "token rows staged");
  static constexpr int KB_BYTES = (BN + MT * XR) * 128;  // one 64-k block of weights + tokens
  static constexpr int KBS = KB_BYTES <= 8192 ? 4 : (KB_BYTES <= 24576 ? 2 : 1);
  static constexpr int X_BYTES = KBS * MT * XR * 128;   // token slabs first in a stage
  static constexpr int W_BYTES = KBS * BN * 128;
  static constexpr int STAGE_BYTES = X_BYTES + W_BYTES;
  // the MMA reads 128 token rows from a 32-row slab: keep that span inside the allocation
  static constexpr int PAD = XR < TC_TILE_M ? (TC_TILE_M - XR) * 128 : 0;
  static constexpr int BUDGET = (CPS == 2 ? 112 : 222) * 1024;
  static constexpr int STAGES = (BUDGET - PAD) / STAGE_BYTES;
  static_assert(STAGES >= 2, "ring too shallow");
  static constexpr int SMEM = STAGES * STAGE_BYTES + PAD + 1024;
  static constexpr int ACC_COLS = KS * MT * BN;  // set j, token tile t at column (j MT + t) BN
  static constexpr int ACC_BUFS = 2 * ACC_COLS <= 512 / CPS ? 2 : 1;
  static constexpr int TMEM_COLS_RAW = ACC_BUFS * ACC_COLS;
  static constexpr int TMEM_COLS =
      TMEM_COLS_RAW <= 32 ? 32 : TMEM_COLS_RAW <= 64 ? 64 : TMEM_COLS_RAW <= 128 ? 128 : TMEM_COLS_RAW <= 256 ? 256 : 512;
  static_assert(TMEM_COLS * CPS <= 512, "TMEM");
};

// Epilogue of the fused QKV projection (bf16 mode): RoPE on the q and k rows
// (stored in the paired order: in every 32-row block of a head, rows 0..15 are
// elements 16b..16b+15 and rows 16..31 their rotate-half partners), q written
// in the activation dtype, k and v appended to the KV cache.
constexpr int EPI_ROPE = BI_EPI_ROPE_KV_APPEND;
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

struct TcArgs {
  void* y;
  int ldy, y_f32, vec_ok;  // vec_ok: y and ldy allow 16-byte stores
  int M, N, K;
  int m_groups, n_groups, splits;
  int m_band;              // token groups per band of the work order (see decode_item)
  float* partial;          // FAST split-K: [splits][M][N] fp32
  const int* mcount;       // optional device row count (rows >= *mcount * mmult are not computed)
  int mmult;
  RopeEpi re;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  return (uint32_t)f32_to_bf16_bits(a) | ((uint32_t)f32_to_bf16_bits(b) << 16);
}
// n consecutive values (n % 8 == 0) to row-contiguous storage.
__device__ __forceinline__ void store_row(void* base, size_t off, const float* v, int n, int f32, int vec_ok) {
  if (vec_ok) {
    if (f32) {
      float4* p = reinterpret_cast<float4*>(reinterpret_cast<float*>(base) + off);
      for (int i = 0; i < n / 4; ++i) p[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    } else {
      uint4* p = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(base) + off);
      for (int i = 0; i < n / 8; ++i)
        p[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                          pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
    }
  } else {
    for (int i = 0; i < n; ++i) store_act(base, off + i, v[i], f32);
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

template <int BN, int MT, int XR, int KS, int EPI, int CPS>
__global__ void __launch_bounds__(TC_THREADS, CPS)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, const TcArgs a) {
  using C = TcCfg<BN, MT, XR, KS, CPS>;
  static_assert(KS == 1 || KS == 2 || KS == 4, "accumulator sets");
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[C::STAGES];
  __shared__ __align__(8) uint64_t empty_bar[C::STAGES];
  __shared__ __align__(8) uint64_t acc_full[2];
  __shared__ __align__(8) uint64_t acc_empty[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int dead_s;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int nkb = a.K / TC_BK;                       // 64-k blocks
  const int kstages_total = (nkb + C::KBS - 1) / C::KBS;  // the last stage may hold fewer k-blocks
  const int ks_per_split = (kstages_total + a.splits - 1) / a.splits;
  const int n_items = a.splits * a.n_groups * a.m_groups;
  // Work item -> (split, weight group, token group).  The token groups are cut
  // into bands of m_band groups; a band's items run weight group by weight
  // group, token group fastest, so the CTAs running together share weight
  // tiles, and a band's token rows (sized to stay in L2) are read from DRAM
  // once instead of once per weight group.  With a device row count: token
  // group slowest, so the live first token group is spread over every CTA.
  const bool mg_major = a.mcount != nullptr;
  auto decode_item = [&](int item, int& sp, int& g, int& mg) {
    if (mg_major) {
      g = item % a.n_groups;
      sp = (item / a.n_groups) % a.splits;
      mg = item / (a.n_groups * a.splits);
    } else {
      const int per_split = a.m_groups * a.n_groups;
      sp = item / per_split;
      const int r = item - sp * per_split;
      const int band = r / (a.m_band * a.n_groups);
      const int m0 = band * a.m_band;
      const int span = min(a.m_band, a.m_groups - m0);
      const int w = r - band * a.m_band * a.n_groups;
      mg = m0 + w % span;
      g = w / span;
    }
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(&drain_bar, 1);
    dead_s = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tmW);
      prefetch_tmap(&tmX);
      int pre = 0;
      if ((int)blockIdx.x < n_items) {
        int sp, g, mg;
        decode_item(blockIdx.x, sp, g, mg);
        if (!mg_major || mg == 0) {
          const int ks0 = sp * ks_per_split, ks1 = min(kstages_total, ks0 + ks_per_split);
          pre = max(0, min(C::STAGES, ks1 - ks0));
          for (int s = 0; s < pre; ++s) {
            mbar_arrive_expect_tx(&full_bar[s], C::STAGE_BYTES);
            tma_load_3d(smem + s * C::STAGE_BYTES + C::X_BYTES, &tmW, 0, g * BN, (ks0 + s) * C::KBS, &full_bar[s]);
          }
        }
      }
      pdl_wait();
      pdl_trigger();
      const int Me = a.mcount ? min(a.M, *a.mcount * a.mmult) : a.M;
      int issued = pre;  // loads issued into the ring so far (slot = n % STAGES, phase = (n / STAGES) & 1)
      int stage = 0;
      uint32_t phase = 0;
      bool first = true;
      if (pre > 0 && Me <= 0) {
        // Nothing to compute: complete the prefetched stages' barriers with
        // their token slabs (zero-filled or in bounds), then drain below.
        int sp, g, mg;
        decode_item(blockIdx.x, sp, g, mg);
        for (int s = 0; s < pre; ++s)
          tma_load_3d(smem + s * C::STAGE_BYTES, &tmX, 0, 0, (sp * ks_per_split + s) * C::KBS, &full_bar[s]);
      } else {
        for (int item = blockIdx.x; item < n_items && !dead_s; item += gridDim.x) {
          int sp, g, mg;
          decode_item(item, sp, g, mg);
          if (mg * MT * TC_TILE_M >= Me) continue;
          const int ks0 = sp * ks_per_split, ks1 = min(kstages_total, ks0 + ks_per_split);
          for (int ks = ks0; ks < ks1; ++ks) {
            uint8_t* sb = smem + stage * C::STAGE_BYTES;
            if (!(first && ks - ks0 < pre)) {
              if (!mbar_wait(&empty_bar[stage], phase ^ 1, SITE_GEMM_EMPTY | (EPI << 12))) {
                dead_s = 1;
                break;
              }
              mbar_arrive_expect_tx(&full_bar[stage], C::STAGE_BYTES);
              tma_load_3d(sb + C::X_BYTES, &tmW, 0, g * BN, ks * C::KBS, &full_bar[stage]);
              ++issued;
            }
            tma_load_3d(sb, &tmX, 0, mg * MT * TC_TILE_M, ks * C::KBS, &full_bar[stage]);
            if (++stage == C::STAGES) {
              stage = 0;
              phase ^= 1;
            }
          }
          first = false;
        }
      }
      if (dead_s || (pre > 0 && Me <= 0)) {
        // No copy may still be writing shared memory when the CTA exits: wait
        // (bounded) for the latest load issued into each slot.
        for (int n = max(0, issued - C::STAGES); n < issued; ++n)
          (void)mbar_wait(&full_bar[n % C::STAGES], (uint32_t)((n / C::STAGES) & 1), SITE_GEMM_DRAIN);
      }
    }
    return;
  }

  if (warp == 5) {
    // ------------------------------------------------------------ TMEM + MMA issuer
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_s)),
                 "n"(C::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    tc_fence_before();
    asm volatile("bar.sync 1, 160;" ::: "memory");
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    pdl_wait();
    pdl_trigger();
    if (lane == 0) {
      const int Me = a.mcount ? min(a.M, *a.mcount * a.mmult) : a.M;
      constexpr uint32_t IDESC = umma_idesc_bf16(TC_TILE_M, BN);
      int stage = 0;
      uint32_t phase = 0;
      int abuf = 0, nacc = 0;
      bool issued_any = false;
      for (int item = blockIdx.x; item < n_items && !dead_s; item += gridDim.x) {
        int sp, g, mg;
        decode_item(item, sp, g, mg);
        if (mg * MT * TC_TILE_M >= Me) continue;
        if (nacc >= C::ACC_BUFS &&
            !mbar_wait(&acc_empty[abuf], (uint32_t)(((nacc / C::ACC_BUFS) - 1) & 1), SITE_GEMM_EMPTY | 0x800)) {
          dead_s = 1;
          break;
        }
        tc_fence_after();
        const int ks0 = sp * ks_per_split, ks1 = min(kstages_total, ks0 + ks_per_split);
        const uint32_t dcol = tmem + abuf * C::ACC_COLS;
        bool ok = true;
        for (int ks = ks0; ks < ks1; ++ks) {
          if (!mbar_wait(&full_bar[stage], phase, SITE_GEMM_FULL | (EPI << 12))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sb = smem_u32(smem + stage * C::STAGE_BYTES);
          const int kbn = min(C::KBS, nkb - ks * C::KBS);
          for (int kb = 0; kb < kbn; ++kb) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t bdesc = umma_sdesc_sw128(sb + C::X_BYTES + kb * (BN * 128) + kk * 32);
#pragma unroll
              for (int j = 0; j < MT; ++j) {
                const uint64_t adesc = umma_sdesc_sw128(sb + kb * (MT * XR * 128) + j * (XR * 128) + kk * 32);
                // k16 step kk of the block goes to set kk % KS; each set's first step starts it
                umma_bf16(dcol + ((kk % KS) * MT + j) * BN, adesc, bdesc, IDESC,
                          (ks > ks0 || kb > 0 || kk >= KS) ? 1u : 0u);
              }
            }
          }
          issued_any = true;
          umma_commit(&empty_bar[stage]);  // the stage is free once these MMAs have read it
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) {
          dead_s = 1;
          break;
        }
        umma_commit(&acc_full[abuf]);  // the accumulator is complete once every MMA so far has finished
        ++nacc;
        abuf = (abuf + 1) % C::ACC_BUFS;
      }
      if (dead_s && issued_any) {  // every MMA issued must finish before TMEM is freed
        umma_commit(&drain_bar);
        (void)mbar_wait(&drain_bar, 0u, SITE_GEMM_DRAIN | 0x800);
      }
    }
    __syncwarp();
    tc_fence_before();
    asm volatile("bar.sync 1, 160;" ::: "memory");
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(C::TMEM_COLS));
    return;
  }

  // -------------------------------------------------------------- epilogue warps 0..3
  asm volatile("bar.sync 1, 160;" ::: "memory");
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  pdl_wait();
  pdl_trigger();
  const int Me = a.mcount ? min(a.M, *a.mcount * a.mmult) : a.M;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  int abuf = 0, nacc = 0;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    int sp, g, mg;
    decode_item(item, sp, g, mg);
    if (mg * MT * TC_TILE_M >= Me) continue;
    if (dead_s) break;
    if (!mbar_wait(&acc_full[abuf], (uint32_t)((nacc / C::ACC_BUFS) & 1), SITE_GEMM_FULL | 0x800)) {
      dead_s = 1;
      break;
    }
    tc_fence_after();
#pragma unroll 1
    for (int j = 0; j < MT; ++j) {
      const int mrow0 = (mg * MT + j) * TC_TILE_M + warp * 32;  // this warp's first token row
      if (mrow0 >= Me) continue;                                // uniform in the warp
      const int m = mrow0 + lane;
      const bool live = m < Me;
#pragma unroll 1
      for (int blk = 0; blk < BN / 32; ++blk) {
        // the KS sets meet in the fixed tree ((s0 + s1) + (s2 + s3)) or s0 + s1
        float v[32];
        const uint32_t col = tmem + lane_base + abuf * C::ACC_COLS + j * BN + blk * 32;
        tmem_ld32(col, v);
        if constexpr (KS >= 2) {
          float u[32];
          tmem_ld32(col + MT * BN, u);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = v[i] + u[i];
        }
        if constexpr (KS == 4) {
          float u[32], t[32];
          tmem_ld32(col + 2 * MT * BN, u);
          tmem_ld32(col + 3 * MT * BN, t);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = v[i] + (u[i] + t[i]);
        }
        if (!live) continue;
        const int n0 = g * BN + blk * 32;  // first weight row of this 32-row block
        if (a.splits > 1) {
          store_row(a.partial, ((size_t)sp * a.M + m) * a.N + n0, v, 32, 1, 1);
        } else if constexpr (EPI == BI_EPI_SWIGLU) {
          float o[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = silu(v[i]) * v[16 + i];
          store_row(a.y, (size_t)m * a.ldy + (n0 >> 1), o, 16, a.y_f32, a.vec_ok);
        } else if constexpr (EPI == EPI_ROPE) {
          const RopeEpi& re = a.re;
          const int QD = re.Hq * re.d, KD = re.Hkv * re.d, half = re.d >> 1;
          const int p = __ldg(re.pos + m), sl = __ldg(re.slot + m);
          if (p < 0 || p >= re.cap || p >= re.table_max_pos || sl < 0 || sl >= re.n_slots) {
            dev_flag(DEVERR_CAPACITY);
            continue;
          }
          if (n0 >= QD + KD) {  // v rows, natural order
            const int ev = n0 - QD - KD;
            const size_t crow = (((size_t)sl * re.n_layers + re.layer) * re.Hkv + ev / re.d) * re.cap + p;
            store_row(re.vc, crow * re.d + ev % re.d, v, 32, 0, 1);
          } else {
            const bool isq = n0 < QD;
            const int rel = isq ? n0 : n0 - QD;
            const int head = rel / re.d, e0 = (rel % re.d) >> 1;  // first-half element 16b
            // cos/sin of the 16 pairs: 128 contiguous bytes of the table row (16-byte loads)
            const float4* tb = reinterpret_cast<const float4*>(re.table + ((size_t)p * half + e0) * 2);
            float ra[16], rb[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 cs = __ldg(tb + i);
              rope_rotate(v[2 * i], v[16 + 2 * i], cs.x, cs.y, ra[2 * i], rb[2 * i]);
              rope_rotate(v[2 * i + 1], v[16 + 2 * i + 1], cs.z, cs.w, ra[2 * i + 1], rb[2 * i + 1]);
            }
            size_t base;
            void* dst;
            if (isq) {
              dst = re.q_out;
              base = (size_t)m * QD + head * re.d;
            } else {
              dst = re.kc;
              base = ((((size_t)sl * re.n_layers + re.layer) * re.Hkv + head) * re.cap + p) * re.d;
            }
            store_row(dst, base + e0, ra, 16, 0, 1);
            store_row(dst, base + e0 + half, rb, 16, 0, 1);
          }
        } else {
          store_row(a.y, (size_t)m * a.ldy + n0, v, 32, a.y_f32, a.vec_ok);
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&acc_empty[abuf]);
    ++nacc;
    abuf = (abuf + 1) % C::ACC_BUFS;
  }
  tc_fence_before();
  asm volatile("bar.sync 1, 160;" ::: "memory");
}

}  // namespace bi
