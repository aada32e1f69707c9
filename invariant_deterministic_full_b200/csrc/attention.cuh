// bi_attention kernels: causal GQA softmax attention on an absolute KV-chunk grid.
//
// Fixed reduction order ("Meituan bitwise train/infer consistency": the
// attention score sum and the softmax denominator are among the reductions
// whose order must be one and the same in Prefill and Decode):
//   * keys are cut on the absolute grid [c*CH, (c+1)*CH), CH = 256 for the
//     invariant variant, whatever the batch or prefill chunking;
//   * score s_j = scale * (q . k_j), the dot product a sequential fp32 FMA
//     chain over the head dimension in ascending order;
//   * chunk max m: exact (any order gives the same max);
//   * chunk denominator l = sum_j exp(s_j - m): lane i of a warp sums keys
//     i, i+32, ..., i+224 in ascending order (masked keys add exactly 0), then
//     a fixed xor-butterfly over the 32 lanes;
//   * chunk numerator acc[e] = sum_j p_j v_j[e]: the keys form 4 interleaved
//     groups (j % 4); each group is a sequential FMA chain over its valid keys
//     in ascending order, and the group sums are added as ((g0+g1)+(g2+g3))
//     (keys past the query add exact zeros, so the sums are the same whether
//     later queries share the tile or not);
//   * merge over chunks 0..pos/CH: M = max m_c, L = sum_c l_c exp(m_c - M),
//     o = sum_c acc_c exp(m_c - M), all in ascending chunk order; out = o / L.
// Those are the CUDA-core kernel's sums (f32 KV, or head size 64).  The
// tensor-core kernels (bf16 KV, head size 128) keep the chunk grid and the
// merge, and differ in three sums:
//   * the denominator: lane i sums keys 8i, ..., 8i+7 in ascending order, then
//     the same xor-butterfly (so each lane's probabilities are contiguous);
//   * the score is eight mma.sync m16n8k16 steps over the head dimension in
//     ascending order, each adding 16 exact products into the (key, pair)
//     fp32 accumulator;
//   * the numerator splits every p exactly into three bf16 parts; each part's
//     products with V accumulate in fp32 over the chunk's keys in ascending
//     16-key steps, and the parts are added as (a0 + a1) + a2.
// Which kernel runs depends on the KV dtype and head size alone, so prefill
// and decode always share one.
// A query's result depends only on its q and the cache rows 0..pos it reads.
#pragma once
#include "common.cuh"

namespace bi {

constexpr int ATT_THREADS = 256;
constexpr int ATT_CHUNK = BI_ATTN_CHUNK;  // 256
constexpr int ATT_MAX_PAIRS = 32;         // (query, q-head) pairs per CTA
constexpr int ATT_MAX_BLOCKS = 1024;      // query blocks per launch
constexpr int ATT_TOKEN_GROUP = 1024;     // tokens per partials workspace pass
constexpr int ATT_MAX_QB = 64;            // tokens per query block

struct AttnPlan {
  int n;
  int2 blk[ATT_MAX_BLOCKS];  // (first token, number of tokens); tokens of a block share the slot, consecutive positions
};

struct AttnArgs {
  const void* q;            // [T][Hq*d] activation dtype
  const int32_t* slot;      // [T]
  const int32_t* pos;       // [T]
  float* part;              // [Tg][Hq][max_chunks][d+4]: acc[d], m, l
  int t_base;               // first token of this group
  int Hq, Hkv, G, d, chunk, max_chunks, layer, n_layers, cap, f32;
  float scale;
  int seg_len;              // chunks per CTA (tensor-core kernel; the CUDA-core kernel takes one)
  int merge_in_cta;         // 1: one segment spans every chunk, the CTA merges and writes out
  int pre_kv;               // 1: slot, pos and every cache row below each token's own position were written by
                            // kernels that completed before the previous launch (a decode step with one token per
                            // slot): attn_dec_kernel reads them and copies its first K sub-tiles before its
                            // dependency wait
  void* out;                // [T][Hq*d] attention output (activation dtype)
};

// Fixed ascending merge of one (query, q head)'s chunk partials 0..nc-1; lane
// l owns head elements l, l+32, ...  The same code serves the merge kernel
// and the attention CTAs that computed all chunks of their queries, so the
// two routes give the same bits.
__device__ __forceinline__ void merge_pair(const float* __restrict__ base, int nc, int d, int lane,
                                           void* __restrict__ out, size_t off, int f32) {
  constexpr int NCR = 4;  // up to NCR chunks: every operand is loaded first, then the same arithmetic runs
  if (nc <= NCR) {
    float mc[NCR], lc[NCR], ac[NCR][4];
#pragma unroll
    for (int c = 0; c < NCR; ++c) {
      if (c < nc) {
        const float* rec = base + (size_t)c * (d + 4);
        mc[c] = rec[d];
        lc[c] = rec[d + 1];
#pragma unroll
        for (int k = 0; k < 4; ++k) ac[c][k] = k < d / 32 ? rec[lane + 32 * k] : 0.f;
      }
    }
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < NCR; ++c)
      if (c < nc) M = fmaxf(M, mc[c]);
    float L = 0.f;
    float o[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < NCR; ++c) {
      if (c < nc) {
        const float w = expf(mc[c] - M);
        L = fmaf(lc[c], w, L);
#pragma unroll
        for (int k = 0; k < 4; ++k) o[k] = fmaf(ac[c][k], w, o[k]);
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (k < d / 32) store_act(out, off + lane + 32 * k, o[k] / L, f32);
    return;
  }
  float M = -INFINITY;
  for (int c = 0; c < nc; ++c) M = fmaxf(M, base[(size_t)c * (d + 4) + d]);
  float L = 0.f;
  float o[4] = {0.f, 0.f, 0.f, 0.f};
  const int ne = d / 32;
  for (int c = 0; c < nc; ++c) {
    const float* rec = base + (size_t)c * (d + 4);
    const float w = expf(rec[d] - M);
    L = fmaf(rec[d + 1], w, L);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (k < ne) o[k] = fmaf(rec[lane + 32 * k], w, o[k]);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (k < ne) store_act(out, off + lane + 32 * k, o[k] / L, f32);
}

__host__ __device__ inline int att_ninner(int d, int f32) { return d * (f32 ? 4 : 2) / 128; }

constexpr int ATT_SUB = 64;  // keys per TMA sub-tile
// sub-tile ring depth: deeper for the small pair groups of decode, whose
// CTAs are short and latency-bound; 2 for the large groups of prefill.
__host__ __device__ constexpr int att_ring(int np) { return np <= 8 ? 4 : 2; }

__host__ __device__ inline size_t att_sub_bytes(int d, int f32) { return (size_t)ATT_SUB * d * (f32 ? 4 : 2); }
__host__ __device__ inline size_t att_smem_bytes(int np, int d, int f32) {
  return att_ring(np) * att_sub_bytes(d, f32) + (size_t)np * d * 4 + 2 * (size_t)np * ATT_CHUNK * 4 + 1024;
}

// Grid: (block, chunk, kv head).  The chunk's K rows, then its V rows, stream
// through a ring of two 64-key sub-tiles (TMA, 128-byte swizzle).  A block's
// (query, head) pairs p = i*G + g (head hk*G + g) are processed NP at a time;
// each group re-streams the chunk (an L2 hit after the first).  Work layout:
//   scores  thread t: key 64*st + (t % 64), pairs (t / 64) + 4k
//   softmax warp w: pairs w, w + 8, ...; lane i: keys i + 32k
//   PV      thread t: element t % d, pairs t / d + (256/d) k
// None of it changes a pair's arithmetic, which is fixed as described above.
template <int NP>
__global__ void __launch_bounds__(ATT_THREADS)
    attn_partial_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ AttnPlan plan, const AttnArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  constexpr int ATT_RING = att_ring(NP);
  __shared__ __align__(8) uint64_t bar[ATT_RING];
  __shared__ float m_s[NP], l_s[NP];
  __shared__ int live_s[NP];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int b = blockIdx.x, c = blockIdx.y, hk = blockIdx.z;
  if (b >= plan.n) return;
  const int t0 = plan.blk[b].x, nq = plan.blk[b].y;
  const int s = a.slot[t0];
  const int pmax = a.pos[t0 + nq - 1];
  const int key0 = c * a.chunk;
  if (key0 > pmax) return;  // chunk beyond every query of the block
  const int nvalid = min(a.chunk, pmax - key0 + 1);
  const int nsub = (nvalid + ATT_SUB - 1) / ATT_SUB;
  const int ninner = att_ninner(a.d, a.f32);
  const int esz = a.f32 ? 4 : 2;
  const size_t sub_bytes = att_sub_bytes(a.d, a.f32);
  float* qs = reinterpret_cast<float*>(smem + ATT_RING * sub_bytes);
  float* S = qs + NP * a.d;       // scores [NP][256]
  float* PT = S + NP * ATT_CHUNK;  // probabilities, key-major [256][NP] (S and PT also host the PV combine)
  const int npairs = nq * a.G;
  const int row_base = ((s * a.n_layers + a.layer) * a.Hkv + hk) * a.cap + key0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nloads = 2 * nsub;  // K sub-tiles then V sub-tiles, per pair group

  if (tid == 0) {
    for (int r = 0; r < ATT_RING; ++r) mbar_init(&bar[r], 1);
    fence_mbar_init();
  }
  __syncthreads();
  // load number L (counted over the whole CTA): sub-tile L % nloads of the
  // sequence K0..K(nsub-1), V0..V(nsub-1), into ring buffer L % ATT_RING.
  auto issue = [&](int L) {
    const int li = L % nloads;
    const bool isv = li >= nsub;
    const int st = isv ? li - nsub : li;
    uint8_t* buf = smem + (L % ATT_RING) * sub_bytes;
    uint64_t* br = &bar[L % ATT_RING];
    mbar_arrive_expect_tx(br, (uint32_t)(ninner * ATT_SUB * 128));
    // one 3-D box {128 bytes, 64 rows, ninner}: lands as ninner swizzled [64][128 B] slabs
    tma_load_3d(buf, isv ? &tmV : &tmK, 0, row_base + st * ATT_SUB, 0, br);
  };
  const int ngroups = (npairs + NP - 1) / NP;
  const int total_loads = ngroups * nloads;
  if (tid == 0)
    for (int L = 0; L < ATT_RING && L < total_loads; ++L) issue(L);
  int L = 0;  // next load to consume
  auto consume_wait = [&]() -> bool { return mbar_wait(&bar[L % ATT_RING], (uint32_t)((L / ATT_RING) & 1), SITE_ATTN_CORE); };
  auto release = [&]() {  // every thread is done with load L: refill its buffer
    __syncthreads();
    if (tid == 0 && L + ATT_RING < total_loads) issue(L + ATT_RING);
    ++L;
  };

  for (int pg0 = 0; pg0 < npairs; pg0 += NP) {
    const int gp = min(NP, npairs - pg0);
    for (int idx = tid; idx < gp * a.d; idx += ATT_THREADS) {
      const int pl = idx / a.d, e = idx % a.d;
      const int p = pg0 + pl;
      const int i = p / a.G, g = p % a.G;
      qs[pl * a.d + e] = load_act(a.q, (size_t)(t0 + i) * a.Hq * a.d + (hk * a.G + g) * a.d + e, a.f32);
    }
    __syncthreads();

    // ---- scores: s = scale * (q . k_j), a sequential fp32 FMA chain over e ascending
    const int pq = tid >> 6;
    for (int st = 0; st < nsub; ++st) {
      if (!consume_wait()) return;
      const int jl = tid & 63;
      const int j = st * ATT_SUB + jl;
      if (j < nvalid) {
        const uint8_t* kb = smem + (L % ATT_RING) * sub_bytes;
        float acc[NP / 4];
#pragma unroll
        for (int k = 0; k < NP / 4; ++k) acc[k] = 0.f;
        const int nch = a.d * esz / 16;
        for (int ch = 0; ch < nch; ++ch) {
          const int ib = ch >> 3, cc = ch & 7;
          const uint4 u = *reinterpret_cast<const uint4*>(kb + ib * (ATT_SUB * 128) + jl * 128 + ((cc ^ (jl & 7)) << 4));
          if (a.f32) {
            const float kv[4] = {__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z),
                                 __uint_as_float(u.w)};
#pragma unroll
            for (int k = 0; k < NP / 4; ++k) {
              const int p = pq + 4 * k;
              if (p < gp) {
                const float4 q0 = *reinterpret_cast<const float4*>(qs + p * a.d + ch * 4);
                float x = acc[k];
                x = fmaf(q0.x, kv[0], x); x = fmaf(q0.y, kv[1], x); x = fmaf(q0.z, kv[2], x); x = fmaf(q0.w, kv[3], x);
                acc[k] = x;
              }
            }
          } else {
            const float kv[8] = {bf16lo(u.x), bf16hi(u.x), bf16lo(u.y), bf16hi(u.y),
                                 bf16lo(u.z), bf16hi(u.z), bf16lo(u.w), bf16hi(u.w)};
#pragma unroll
            for (int k = 0; k < NP / 4; ++k) {
              const int p = pq + 4 * k;
              if (p < gp) {
                const float* qp = qs + p * a.d + ch * 8;
                const float4 q0 = *reinterpret_cast<const float4*>(qp);
                const float4 q1 = *reinterpret_cast<const float4*>(qp + 4);
                float x = acc[k];
                x = fmaf(q0.x, kv[0], x); x = fmaf(q0.y, kv[1], x); x = fmaf(q0.z, kv[2], x); x = fmaf(q0.w, kv[3], x);
                x = fmaf(q1.x, kv[4], x); x = fmaf(q1.y, kv[5], x); x = fmaf(q1.z, kv[6], x); x = fmaf(q1.w, kv[7], x);
                acc[k] = x;
              }
            }
          }
        }
#pragma unroll
        for (int k = 0; k < NP / 4; ++k) {
          const int p = pq + 4 * k;
          if (p < gp) S[p * ATT_CHUNK + j] = acc[k] * a.scale;
        }
      }
      release();
    }

    // ---- softmax per pair: max (exact), exp, l = per-lane ascending sums then fixed butterfly
    for (int pl = warp; pl < gp; pl += ATT_THREADS / 32) {
      const int i = (pg0 + pl) / a.G;
      const int lim = a.pos[t0 + i] - key0;  // keys j <= lim are visible to this query
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < ATT_CHUNK / 32; ++k) {
        const int j = lane + 32 * k;
        if (j <= lim && j < nvalid) mx = fmaxf(mx, S[pl * ATT_CHUNK + j]);
      }
      mx = warp_max(mx);
      float sum = 0.f;
#pragma unroll
      for (int k = 0; k < ATT_CHUNK / 32; ++k) {
        const int j = lane + 32 * k;
        float pj = 0.f;
        if (j <= lim && j < nvalid) pj = expf(S[pl * ATT_CHUNK + j] - mx);
        if (j < nvalid) PT[j * NP + pl] = pj;
        sum += pj;
      }
      sum = warp_sum_fixed(sum);
      if (lane == 0) {
        m_s[pl] = mx;
        l_s[pl] = sum;
        live_s[pl] = lim >= 0;
      }
    }
    __syncthreads();

    // ---- PV: acc[e] = sum_j p_j v_j[e].  The keys of the chunk fall into 4
    // interleaved groups (j % 4); each group is summed with sequential FMAs in
    // ascending j, and the group sums are combined as ((g0 + g1) + (g2 + g3)).
    // Thread t: key group t / 64, element pair ep, all pairs of its phase.
    const int kg = tid >> 6;
    const int r64 = tid & 63;
    const int nep = a.d / 2;           // element pairs per row (64 or 32)
    const int ep = r64 % nep;
    const int ph = r64 / nep;          // pair phase (d = 64: pairs ph, ph + 2, ...)
    const int pst = 64 / nep;          // pair stride: 1 (d = 128) or 2 (d = 64)
    const int ebyte = ep * 2 * esz;
    const int ib_e = ebyte >> 7, cc_e = (ebyte & 127) >> 4, within = ebyte & 15;
    float pacc[NP][2];
#pragma unroll
    for (int k = 0; k < NP; ++k) pacc[k][0] = pacc[k][1] = 0.f;
    for (int st = 0; st < nsub; ++st) {
      if (!consume_wait()) return;
      const uint8_t* vb = smem + (L % ATT_RING) * sub_bytes + ib_e * (ATT_SUB * 128) + within;
      const int jend = min(ATT_SUB, nvalid - st * ATT_SUB);
      for (int jl = kg; jl < jend; jl += 4) {
        const uint8_t* vp = vb + jl * 128 + ((cc_e ^ (jl & 7)) << 4);
        float v0, v1;
        if (a.f32) {
          const float2 vv = *reinterpret_cast<const float2*>(vp);
          v0 = vv.x;
          v1 = vv.y;
        } else {
          const uint32_t vv = *reinterpret_cast<const uint32_t*>(vp);
          v0 = bf16lo(vv);
          v1 = bf16hi(vv);
        }
        const float* pr = PT + (st * ATT_SUB + jl) * NP;
        if (pst == 1) {
#pragma unroll
          for (int k = 0; k < NP; ++k) {
            const float pv = pr[k];
            pacc[k][0] = fmaf(pv, v0, pacc[k][0]);
            pacc[k][1] = fmaf(pv, v1, pacc[k][1]);
          }
        } else {
#pragma unroll
          for (int k = 0; k < NP / 2; ++k) {
            const float pv = pr[ph + 2 * k];
            pacc[k][0] = fmaf(pv, v0, pacc[k][0]);
            pacc[k][1] = fmaf(pv, v1, pacc[k][1]);
          }
        }
      }
      release();
    }
    // combine the 4 key groups in a fixed tree (S and PT are free: reuse them)
    float* red = S;  // [4][NP][d]
#pragma unroll
    for (int k = 0; k < NP; ++k) {
      const int pl = ph + k * pst;
      if (k < NP / pst) {
        red[(kg * NP + pl) * a.d + 2 * ep] = pacc[k][0];
        red[(kg * NP + pl) * a.d + 2 * ep + 1] = pacc[k][1];
      }
    }
    __syncthreads();
    for (int idx = tid; idx < gp * a.d; idx += ATT_THREADS) {
      const int pl = idx / a.d, e = idx % a.d;
      if (!live_s[pl]) continue;
      const float o = (red[(0 * NP + pl) * a.d + e] + red[(1 * NP + pl) * a.d + e]) +
                      (red[(2 * NP + pl) * a.d + e] + red[(3 * NP + pl) * a.d + e]);
      const int p = pg0 + pl;
      const int i = p / a.G, g = p % a.G;
      const int hq = hk * a.G + g;
      float* rec = a.part + (((size_t)(t0 + i - a.t_base) * a.Hq + hq) * a.max_chunks + c) * (a.d + 4);
      rec[e] = o;
      if (e == 0) {
        rec[a.d] = m_s[pl];
        rec[a.d + 1] = l_s[pl];
      }
    }
    __syncthreads();  // the next group overwrites q, S and the pair statistics
  }
}

// ---------------------------------------------------------------------------
// bf16 mode on tensor cores (mma.sync m16n8k16, fp32 accumulate).  The same
// chunk grid, masks and max as above; the denominator and the probabilities
// come from atc_softmax_row (eight contiguous keys per lane).  The
// (query, q head) pairs are the 8-column side of every mma, so a decode group
// of G <= 8 pairs fills at least half a tile:
//   * scores  S^T[key][pair] = scale * sum_d K[key][d] q[pair][d]
//     (A = K tile, B = q^T): one chain of 8 ascending k16 steps over the head
//     dimension per element (bf16 x bf16 products are exact);
//   * output  O^T[e][pair] = sum_key V[key][e] P[pair][key]
//     (A = V^T tile, B = P^T): the fp32 probabilities are split exactly into
//     three bf16 parts P = P0 + P1 + P2 (8+8+8 significant bits), each part's
//     product accumulated over ascending k16 steps of keys in its own fp32
//     accumulator, and the three added as (o0 + o1) + o2.
// Column p of an mma result depends only on column p of its B operand, so a
// pair's result does not depend on how many pairs share the tile -- decode
// (8- or 16-pair groups) and prefill (32-pair groups) give the same bits.
// Pair rows past the group are never computed or stored.  Keys past a query
// have P = 0 and add exact zeros; V rows past the last valid key are zeroed in
// shared memory before use.
constexpr int ATC_SST = 260;  // row stride of the fp32 score tile (floats): conflict-free fragment stores

__host__ __device__ inline size_t atc_smem_bytes(int npt, int ring) {
  const size_t np = 8 * npt;
  return (size_t)ring * 16384      // K/V sub-tiles: [2 halves][64 keys][128 B]
         + np * 256                // q tile: [2 halves][np][128 B]
         + np * ATC_SST * 4        // scores [np][ATC_SST]
         + 3 * np * 512            // probability parts [3][np][256 keys] bf16, 16-byte chunks swizzled
         + 1024;
}

// byte offset of key j of pair row r in a probability part
__device__ __forceinline__ uint32_t atc_poff(int r, int j) {
  const int c = j >> 3;
  return (uint32_t)(r * 512 + (((c & ~7) | ((c ^ r) & 7)) << 4) + (j & 7) * 2);
}

// Softmax of one (pair, chunk) row of scores, the one sequence every
// tensor-core schedule runs: lane l owns keys 8l .. 8l+7 of the chunk (two
// 16-byte score loads); max over the visible keys (exact); each lane sums its
// eight exp(s - max) in ascending key order, then the fixed xor-butterfly;
// every probability is split exactly into three bf16 parts, stored as one
// 16-byte vector per part at row pl of each part (zeros past the visible
// keys).  srow: the row's 256 scores (16-byte aligned); part q of the
// probabilities at pbase + q * part_bytes.
__device__ __forceinline__ void atc_softmax_row(const float* __restrict__ srow, uint8_t* __restrict__ pbase,
                                                int part_bytes, int pl, int lim, int nvalid, int lane, float& mx_out,
                                                float& sum_out) {
  const int j0 = lane * 8;
  const float4 sa = *reinterpret_cast<const float4*>(srow + j0), sb = *reinterpret_cast<const float4*>(srow + j0 + 4);
  const float sv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
  float mx = -INFINITY;
#pragma unroll
  for (int e = 0; e < 8; ++e)
    if (j0 + e <= lim && j0 + e < nvalid) mx = fmaxf(mx, sv[e]);
  mx = warp_max(mx);
  float sum = 0.f;
  uint32_t w[3][4];
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    uint16_t q[3][2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = j0 + e + h;
      float pj = 0.f;
      if (j <= lim && j < nvalid) pj = expf(sv[e + h] - mx);
      sum += pj;
      q[0][h] = f32_to_bf16_bits(pj);
      const float r0 = pj - bf16_bits_to_f32(q[0][h]);
      q[1][h] = f32_to_bf16_bits(r0);
      q[2][h] = f32_to_bf16_bits(r0 - bf16_bits_to_f32(q[1][h]));
    }
#pragma unroll
    for (int t = 0; t < 3; ++t) w[t][e >> 1] = (uint32_t)q[t][0] | ((uint32_t)q[t][1] << 16);
  }
  const uint32_t off = atc_poff(pl, j0);
#pragma unroll
  for (int t = 0; t < 3; ++t)
    *reinterpret_cast<uint4*>(pbase + t * part_bytes + off) = make_uint4(w[t][0], w[t][1], w[t][2], w[t][3]);
  mx_out = mx;
  sum_out = warp_sum_fixed(sum);
}

constexpr int ATC_THREADS = ATT_THREADS + 32;  // 8 consumer warps + 1 producer warp

template <int NPT, int RING>
__global__ void __launch_bounds__(ATC_THREADS)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ AttnPlan plan, const AttnArgs a) {
  pdl_wait();
  pdl_trigger();
  constexpr int NP = 8 * NPT;  // pairs per group
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[RING];
  __shared__ __align__(8) uint64_t empty_bar[RING];
  __shared__ float m_s[NP], l_s[NP];
  __shared__ int live_s[NP];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int b = blockIdx.x, sg = blockIdx.y, hk = blockIdx.z;
  if (b >= plan.n) return;
  const int t0 = plan.blk[b].x, nq = plan.blk[b].y;
  const int s = a.slot[t0];
  const int pmax = a.pos[t0 + nq - 1];
  // this CTA's segment of the absolute chunk grid, walked in ascending order
  const int c_lo = sg * a.seg_len;
  int c_hi = min(pmax / a.chunk + 1, c_lo + a.seg_len);
  if (c_hi > a.max_chunks) {  // device position beyond what the launch was planned for
    if (threadIdx.x == 0) dev_flag(DEVERR_CAPACITY);
    c_hi = a.max_chunks;
  }
  if (c_lo >= c_hi) return;
  const int npairs = nq * a.G;
  const int cache_base = ((s * a.n_layers + a.layer) * a.Hkv + hk) * a.cap;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  constexpr uint32_t SUB = 16384;
  uint8_t* qt = smem + RING * SUB;                             // [2][NP][128 B]
  float* S = reinterpret_cast<float*>(qt + NP * 256);          // [NP][ATC_SST]
  uint8_t* Pp = reinterpret_cast<uint8_t*>(S + NP * ATC_SST);  // [3][NP][512 B]
  const uint32_t qt_s = smem_u32(qt), pp_s = smem_u32(Pp);
  const int ngroups = (npairs + NP - 1) / NP;
  auto nsub_of = [&](int c) { return (min(a.chunk, pmax - c * a.chunk + 1) + ATT_SUB - 1) / ATT_SUB; };

  if (tid == 0) {
    for (int r = 0; r < RING; ++r) {
      mbar_init(&full_bar[r], 1);
      mbar_init(&empty_bar[r], ATT_THREADS / 32);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == ATT_THREADS / 32) {
    // ---- producer warp, one lane: for each chunk of the segment, for each pair
    // group, the chunk's K sub-tiles then its V sub-tiles.  A slot is refilled
    // once all eight consumer warps have released it, so the stream runs ahead
    // of the slowest warp by up to RING sub-tiles, across chunk boundaries.
    if (lane == 0) {
      int lp = 0;
      for (int pc = c_lo; pc < c_hi; ++pc) {
        const int pns = nsub_of(pc);
        for (int pg = 0; pg < ngroups; ++pg)
          for (int pli = 0; pli < 2 * pns; ++pli, ++lp) {
            const int slot = lp % RING;
            if (lp >= RING && !mbar_wait(&empty_bar[slot], (uint32_t)(((lp / RING) - 1) & 1), SITE_ATTN_TC | 0x80))
              return;
            const bool isv = pli >= pns;
            const int st = isv ? pli - pns : pli;
            mbar_arrive_expect_tx(&full_bar[slot], SUB);
            tma_load_3d(smem + slot * SUB, isv ? &tmV : &tmK, 0, cache_base + pc * a.chunk + st * ATT_SUB, 0,
                        &full_bar[slot]);
          }
      }
    }
    return;
  }

  // ---- consumer warps.  A ring wait that runs out sets the error flag; the warp
  // then goes on (on stale data) so every named barrier is still met.
  int L = 0;
  auto consume_wait = [&]() {
    (void)mbar_wait(&full_bar[L % RING], (uint32_t)((L / RING) & 1), SITE_ATTN_TC | (NPT << 8));
  };
  auto release = [&]() {  // this warp is done with slot L
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[L % RING]);
    ++L;
  };
  auto cbar = []() { asm volatile("bar.sync 1, %0;" ::"n"(ATT_THREADS) : "memory"); };

  // score work of a warp: key tile kt of each 64-key sub-tile, pair tiles pt = spt, spt + 2, ...
  constexpr int SPT = NPT == 1 ? 1 : NPT / 2;  // pair tiles per warp in the score phase
  const int kt = warp & 3;
  const int spt0 = NPT == 1 ? 0 : (warp >> 2);
  const bool score_warp = NPT > 1 || warp < 4;

  // positions of the block's queries (consecutive tokens of one slot), read once
  __shared__ int pos_s[ATT_MAX_QB];
  for (int i = tid; i < nq; i += ATT_THREADS) pos_s[i] = a.pos[t0 + i];
  // q tile (bf16, 128-byte swizzle per half; padded rows are zero) and the q^T
  // fragments (B operand) of this warp's pair tiles; with one pair group they
  // are loaded once for the whole segment
  uint32_t qb[SPT][8][2];
  auto load_q = [&](int pg0, int gp) {
    for (int idx = tid; idx < NP * 16; idx += ATT_THREADS) {  // 16 chunks of 8 elements per row
      const int row = idx >> 4, ch = idx & 15;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (row < gp) {
        const int p = pg0 + row;
        const int i = p / a.G, g = p % a.G;
        v = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.q) +
                                            (size_t)(t0 + i) * a.Hq * 128 + (hk * a.G + g) * 128 + ch * 8);
      }
      const int half = ch >> 3, cc = ch & 7;
      *reinterpret_cast<uint4*>(qt + half * (NP * 128) + row * 128 + ((cc ^ (row & 7)) << 4)) = v;
    }
    cbar();
    if (score_warp) {
#pragma unroll
      for (int u = 0; u < SPT; ++u)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int row = (spt0 + 2 * u) * 8 + (lane & 7);
          const int half = kk >> 2, ch = 2 * (kk & 3) + ((lane >> 3) & 1);
          ldsm_x2(qt_s + half * (NP * 128) + row * 128 + ((ch ^ (row & 7)) << 4), qb[u][kk][0], qb[u][kk][1]);
        }
    }
  };
  if (ngroups == 1) load_q(0, npairs);

  for (int c = c_lo; c < c_hi; ++c) {
    const int key0 = c * a.chunk;
    const int nvalid = min(a.chunk, pmax - key0 + 1);
    const int nsub = (nvalid + ATT_SUB - 1) / ATT_SUB;
    for (int pg0 = 0; pg0 < npairs; pg0 += NP) {
      const int gp = min(NP, npairs - pg0);
      if (ngroups > 1) load_q(pg0, gp);

      // ---- scores: S[pair][key] = scale * (K[key] . q[pair])
      for (int st = 0; st < nsub; ++st) {
        consume_wait();
        if (score_warp) {
          const uint32_t kb = smem_u32(smem + (L % RING) * SUB);
          float acc[SPT][4];
#pragma unroll
          for (int u = 0; u < SPT; ++u) acc[u][0] = acc[u][1] = acc[u][2] = acc[u][3] = 0.f;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const int krow = kt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
            const int half = kk >> 2, ch = 2 * (kk & 3) + (lane >> 4);
            uint32_t ka[4];
            ldsm_x4(kb + half * 8192 + krow * 128 + ((ch ^ (krow & 7)) << 4), ka[0], ka[1], ka[2], ka[3]);
#pragma unroll
            for (int u = 0; u < SPT; ++u) mma_bf16_16816(acc[u], ka, qb[u][kk][0], qb[u][kk][1]);
          }
#pragma unroll
          for (int u = 0; u < SPT; ++u) {
            const int pr = (spt0 + 2 * u) * 8 + 2 * t4;
            const int j = st * ATT_SUB + kt * 16 + g8;
            S[pr * ATC_SST + j] = acc[u][0] * a.scale;
            S[(pr + 1) * ATC_SST + j] = acc[u][1] * a.scale;
            S[pr * ATC_SST + j + 8] = acc[u][2] * a.scale;
            S[(pr + 1) * ATC_SST + j + 8] = acc[u][3] * a.scale;
          }
        }
        release();
      }
      cbar();  // every score of the chunk is in S

      // ---- softmax of the live pair rows (atc_softmax_row).  Rows past the group's pairs are
      // not computed: they only reach output columns never stored.
      for (int pl = warp; pl < gp; pl += ATT_THREADS / 32) {
        const int i = (pg0 + pl) / a.G;
        const int lim = pos_s[i] - key0;
        float mx, sum;
        atc_softmax_row(S + pl * ATC_SST, Pp, NP * 512, pl, lim, nvalid, lane, mx, sum);
        if (lane == 0) {
          m_s[pl] = mx;
          l_s[pl] = sum;
          live_s[pl] = lim >= 0;
        }
      }
      cbar();

      // ---- P.V: warp w owns head elements 16w..16w+15 (one m16 tile of V^T)
      float pacc[3][NPT][4];
#pragma unroll
      for (int q = 0; q < 3; ++q)
#pragma unroll
        for (int u = 0; u < NPT; ++u) pacc[q][u][0] = pacc[q][u][1] = pacc[q][u][2] = pacc[q][u][3] = 0.f;
      for (int st = 0; st < nsub; ++st) {
        consume_wait();
        uint8_t* vbuf = smem + (L % RING) * SUB;
        const int vrows = nvalid - st * ATT_SUB;  // valid rows of this sub-tile
        if (vrows < ATT_SUB) {  // zero the rows past the last valid key
          for (int idx = tid; idx < (ATT_SUB - vrows) * 16; idx += ATT_THREADS) {
            const int r = vrows + (idx >> 4), ch = idx & 15;
            *reinterpret_cast<uint4*>(vbuf + (ch >> 3) * 8192 + r * 128 + ((ch & 7) << 4)) = make_uint4(0u, 0u, 0u, 0u);
          }
          cbar();
        }
        const uint32_t vb = smem_u32(vbuf);
        const int nk16 = min(4, (vrows + 15) / 16);
        for (int kk = 0; kk < nk16; ++kk) {
          // A fragment: V^T rows = head elements 16w.., columns = keys 16kk.. of the sub-tile
          uint32_t va[4];
          {
            const int krow = kk * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
            const int e0 = warp * 16 + ((lane >> 3) & 1) * 8;
            const int half = e0 >> 6, ch = (e0 & 63) >> 3;
            ldsm_x4_trans(vb + half * 8192 + krow * 128 + ((ch ^ (krow & 7)) << 4), va[0], va[1], va[2], va[3]);
          }
          const int j0 = st * ATT_SUB + kk * 16;  // first key of this k16 step within the chunk
#pragma unroll
          for (int q = 0; q < 3; ++q) {
#pragma unroll
            for (int u = 0; u < NPT; ++u) {
              uint32_t pb0, pb1;
              const int row = u * 8 + (lane & 7);
              ldsm_x2(pp_s + q * (NP * 512) + atc_poff(row, j0 + ((lane >> 3) & 1) * 8), pb0, pb1);
              mma_bf16_16816(pacc[q][u], va, pb0, pb1);
            }
          }
        }
        release();
      }
      // partial record of each live pair: acc[e] = (o0 + o1) + o2, then m and l
#pragma unroll
      for (int u = 0; u < NPT; ++u)
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int pl = u * 8 + 2 * t4 + cc;
          if (pl >= gp || !live_s[pl]) continue;
          const int p = pg0 + pl;
          const int i = p / a.G, g = p % a.G;
          const int hq = hk * a.G + g;
          float* rec = a.part + (((size_t)(t0 + i - a.t_base) * a.Hq + hq) * a.max_chunks + c) * (128 + 4);
          const int e = warp * 16 + g8;
          rec[e] = (pacc[0][u][cc] + pacc[1][u][cc]) + pacc[2][u][cc];
          rec[e + 8] = (pacc[0][u][2 + cc] + pacc[1][u][2 + cc]) + pacc[2][u][2 + cc];
          if (warp == 0 && g8 == 0) {
            rec[128] = m_s[pl];
            rec[129] = l_s[pl];
          }
        }
      cbar();  // the next group overwrites q, S, the probability parts and the statistics
    }
  }
  if (a.merge_in_cta) {
    // every chunk of the block's queries was computed above: merge them here
    // (the partials written by this CTA are visible to it after the barrier)
    for (int p = warp; p < npairs; p += ATT_THREADS / 32) {
      const int t = t0 + p / a.G, hq = hk * a.G + p % a.G;
      const int nc = min(pos_s[t - t0] / a.chunk + 1, c_hi);
      merge_pair(a.part + ((size_t)(t - a.t_base) * a.Hq + hq) * a.max_chunks * (128 + 4), nc, 128, lane, a.out,
                 (size_t)t * a.Hq * 128 + hq * 128, 0);
    }
  }
}

// ---------------------------------------------------------------------------
// Prefill schedule of the same computation (query blocks of up to
// ATT_MAX_QB consecutive tokens; their (query, q head) pairs in groups of 16).
// attn_tc_kernel streams a chunk's K and V rows through its ring once per
// pair group.  Here a CTA keeps the chunk's K rows and V rows resident in
// shared memory (128 KB) and two groups of eight consumer warps run the
// block's pair groups against them, alternately, so that each SM keeps four
// warps per sub-partition busy; the next chunk's K rows are requested once
// both warp groups have their last scores, its V rows once both have done
// their last P.V.  Every score, softmax, P split, P.V chain, record and merge
// is attn_tc_kernel's instruction sequence for the same element, so prefill
// and decode keep giving the same bits.
constexpr int ATP_NP = 16;          // pairs per group
constexpr int ATP_WG = 2;           // consumer warp groups of ATT_THREADS threads
constexpr int ATP_THREADS = ATP_WG * ATT_THREADS + 32;
constexpr size_t ATP_WG_BYTES = 2 * ATP_NP * 128 + (size_t)ATP_NP * ATC_SST * 4 + 3 * ATP_NP * 512;
__host__ __device__ inline size_t atp_smem_bytes() {
  return (size_t)2 * 4 * 16384  // K and V rows of one chunk: 4 sub-tiles each
         + ATP_WG * ATP_WG_BYTES // per warp group: q tile [2][NP][128 B], scores [NP][ATC_SST], P parts [3][NP][512 B]
         + 1024;
}

__global__ void __launch_bounds__(ATP_THREADS, 1)
    attn_pre_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ AttnPlan plan, const AttnArgs a) {
  pdl_wait();
  pdl_trigger();
  constexpr int NP = ATP_NP, NPT = NP / 8, SPT = NPT / 2;
  constexpr int NCW = ATP_WG * ATT_THREADS / 32;  // consumer warps
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_k, full_v, empty_k, empty_v;
  __shared__ float m_s[ATP_WG][NP], l_s[ATP_WG][NP];
  __shared__ int live_s[ATP_WG][NP];
  __shared__ int pos_s[ATT_MAX_QB];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int b = blockIdx.x, sg = blockIdx.y, hk = blockIdx.z;
  if (b >= plan.n) return;
  const int t0 = plan.blk[b].x, nq = plan.blk[b].y;
  const int s = a.slot[t0];
  const int pmax = a.pos[t0 + nq - 1];
  const int c_lo = sg * a.seg_len;
  int c_hi = min(pmax / a.chunk + 1, c_lo + a.seg_len);
  if (c_hi > a.max_chunks) {  // device position beyond what the launch was planned for
    if (threadIdx.x == 0) dev_flag(DEVERR_CAPACITY);
    c_hi = a.max_chunks;
  }
  if (c_lo >= c_hi) return;
  const int npairs = nq * a.G;
  const int ngroups = (npairs + NP - 1) / NP;
  const int cache_base = ((s * a.n_layers + a.layer) * a.Hkv + hk) * a.cap;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  constexpr uint32_t SUB = 16384;
  uint8_t* kbuf = smem;  // [4 sub-tiles][16 KB]
  uint8_t* vbuf = smem + 4 * SUB;
  auto nsub_of = [&](int c) { return (min(a.chunk, pmax - c * a.chunk + 1) + ATT_SUB - 1) / ATT_SUB; };

  if (tid == 0) {
    mbar_init(&full_k, 1);
    mbar_init(&full_v, 1);
    mbar_init(&empty_k, NCW);
    mbar_init(&empty_v, NCW);
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == NCW) {
    // ---- producer warp, one lane: per chunk, its K rows into kbuf, its V rows into vbuf
    if (lane == 0) {
      for (int pc = c_lo; pc < c_hi; ++pc) {
        const int pns = nsub_of(pc);
        const uint32_t par = (uint32_t)((pc - c_lo - 1) & 1);
        for (int isv = 0; isv < 2; ++isv) {
          uint64_t* fb = isv ? &full_v : &full_k;
          if (pc > c_lo && !mbar_wait(isv ? &empty_v : &empty_k, par, SITE_ATTN_TC | 0xA0)) return;
          mbar_arrive_expect_tx(fb, pns * SUB);
          for (int st = 0; st < pns; ++st)
            tma_load_3d((isv ? vbuf : kbuf) + st * SUB, isv ? &tmV : &tmK, 0, cache_base + pc * a.chunk + st * ATT_SUB,
                        0, fb);
        }
      }
    }
    return;
  }

  // ---- consumer warp groups: group wg takes the pair groups gi = wg, wg + ATP_WG, ...
  const int wg = warp / 8, wl = warp % 8;  // warp group, warp within it
  uint8_t* wbase = smem + 8 * SUB + wg * ATP_WG_BYTES;
  uint8_t* qt = wbase;                                         // [2][NP][128 B]
  float* S = reinterpret_cast<float*>(qt + NP * 256);          // [NP][ATC_SST]
  uint8_t* Pp = reinterpret_cast<uint8_t*>(S + NP * ATC_SST);  // [3][NP][512 B]
  const uint32_t qt_s = smem_u32(qt), pp_s = smem_u32(Pp);
  const int gbar = 1 + wg;  // named barrier of the warp group
  auto gsync = [&]() { asm volatile("bar.sync %0, %1;" ::"r"(gbar), "n"(ATT_THREADS) : "memory"); };
  auto csync = []() { asm volatile("bar.sync 3, %0;" ::"n"(NCW * 32) : "memory"); };  // every consumer warp
  const int kt = wl & 3, spt0 = wl >> 2;
  for (int i = tid; i < nq; i += NCW * 32) pos_s[i] = a.pos[t0 + i];
  csync();  // the positions are read by both warp groups
  const int my_last = ngroups > wg ? wg + ((ngroups - 1 - wg) / ATP_WG) * ATP_WG : -1;  // this group's last pair group

  for (int c = c_lo; c < c_hi; ++c) {
    const uint32_t par = (uint32_t)((c - c_lo) & 1);
    const int key0 = c * a.chunk;
    const int nvalid = min(a.chunk, pmax - key0 + 1);
    const int nsub = (nvalid + ATT_SUB - 1) / ATT_SUB;
    (void)mbar_wait(&full_k, par, SITE_ATTN_TC | 0xB0);
    if (my_last < 0) {  // no pair group for this warp group: the chunk's K rows are free at once
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_k);
    }
    bool v_ready = false;
    auto v_prepare = [&]() {  // once per chunk, by every consumer warp: wait for V, zero the rows past the last key
      (void)mbar_wait(&full_v, par, SITE_ATTN_TC | 0xC0);
      const int vpad = nsub * ATT_SUB - nvalid;
      for (int idx = tid; idx < vpad * 16; idx += NCW * 32) {
        const int r = nvalid + (idx >> 4), ch = idx & 15;  // row within the chunk
        *reinterpret_cast<uint4*>(vbuf + (r / ATT_SUB) * SUB + (ch >> 3) * 8192 + (r % ATT_SUB) * 128 +
                                  ((ch & 7) << 4)) = make_uint4(0u, 0u, 0u, 0u);
      }
      csync();
      v_ready = true;
    };
    for (int gi = wg; gi < ngroups; gi += ATP_WG) {
      const int pg0 = gi * NP;
      const int gp = min(NP, npairs - pg0);
      // q tile of the group (bf16, 128-byte swizzle per half; padded rows are zero)
      for (int idx = tid - wg * ATT_THREADS; idx < NP * 16; idx += ATT_THREADS) {
        const int row = idx >> 4, ch = idx & 15;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (row < gp) {
          const int p = pg0 + row;
          const int i = p / a.G, g = p % a.G;
          v = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.q) +
                                              (size_t)(t0 + i) * a.Hq * 128 + (hk * a.G + g) * 128 + ch * 8);
        }
        const int half = ch >> 3, cc = ch & 7;
        *reinterpret_cast<uint4*>(qt + half * (NP * 128) + row * 128 + ((cc ^ (row & 7)) << 4)) = v;
      }
      gsync();
      uint32_t qb[SPT][8][2];
#pragma unroll
      for (int u = 0; u < SPT; ++u)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int row = (spt0 + 2 * u) * 8 + (lane & 7);
          const int half = kk >> 2, ch = 2 * (kk & 3) + ((lane >> 3) & 1);
          ldsm_x2(qt_s + half * (NP * 128) + row * 128 + ((ch ^ (row & 7)) << 4), qb[u][kk][0], qb[u][kk][1]);
        }

      // ---- scores: S[pair][key] = scale * (K[key] . q[pair]), K resident
      for (int st = 0; st < nsub; ++st) {
        const uint32_t kb = smem_u32(kbuf + st * SUB);
        float acc[SPT][4];
#pragma unroll
        for (int u = 0; u < SPT; ++u) acc[u][0] = acc[u][1] = acc[u][2] = acc[u][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int krow = kt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int half = kk >> 2, ch = 2 * (kk & 3) + (lane >> 4);
          uint32_t ka[4];
          ldsm_x4(kb + half * 8192 + krow * 128 + ((ch ^ (krow & 7)) << 4), ka[0], ka[1], ka[2], ka[3]);
#pragma unroll
          for (int u = 0; u < SPT; ++u) mma_bf16_16816(acc[u], ka, qb[u][kk][0], qb[u][kk][1]);
        }
#pragma unroll
        for (int u = 0; u < SPT; ++u) {
          const int pr = (spt0 + 2 * u) * 8 + 2 * t4;
          const int j = st * ATT_SUB + kt * 16 + g8;
          S[pr * ATC_SST + j] = acc[u][0] * a.scale;
          S[(pr + 1) * ATC_SST + j] = acc[u][1] * a.scale;
          S[pr * ATC_SST + j + 8] = acc[u][2] * a.scale;
          S[(pr + 1) * ATC_SST + j + 8] = acc[u][3] * a.scale;
        }
      }
      if (gi == my_last) {  // this warp group's last scores of the chunk: its K rows may be replaced
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_k);
      }
      gsync();  // every score of the group is in S

      // ---- softmax of the live pair rows (attn_tc_kernel's sequence)
      for (int pl = wl; pl < gp; pl += 8) {
        const int i = (pg0 + pl) / a.G;
        const int lim = pos_s[i] - key0;
        float mx, sum;
        atc_softmax_row(S + pl * ATC_SST, Pp, NP * 512, pl, lim, nvalid, lane, mx, sum);
        if (lane == 0) {
          m_s[wg][pl] = mx;
          l_s[wg][pl] = sum;
          live_s[wg][pl] = lim >= 0;
        }
      }
      if (!v_ready) v_prepare();  // both warp groups meet here once per chunk
      gsync();

      // ---- P.V: warp wl owns head elements 16 wl..16 wl + 15 (one m16 tile of V^T), V resident
      float pacc[3][NPT][4];
#pragma unroll
      for (int q = 0; q < 3; ++q)
#pragma unroll
        for (int u = 0; u < NPT; ++u) pacc[q][u][0] = pacc[q][u][1] = pacc[q][u][2] = pacc[q][u][3] = 0.f;
      for (int st = 0; st < nsub; ++st) {
        const uint32_t vb = smem_u32(vbuf + st * SUB);
        const int vrows = nvalid - st * ATT_SUB;
        const int nk16 = min(4, (vrows + 15) / 16);
        for (int kk = 0; kk < nk16; ++kk) {
          uint32_t va[4];
          {
            const int krow = kk * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
            const int e0 = wl * 16 + ((lane >> 3) & 1) * 8;
            const int half = e0 >> 6, ch = (e0 & 63) >> 3;
            ldsm_x4_trans(vb + half * 8192 + krow * 128 + ((ch ^ (krow & 7)) << 4), va[0], va[1], va[2], va[3]);
          }
          const int j0 = st * ATT_SUB + kk * 16;
#pragma unroll
          for (int q = 0; q < 3; ++q) {
#pragma unroll
            for (int u = 0; u < NPT; ++u) {
              uint32_t pb0, pb1;
              const int row = u * 8 + (lane & 7);
              ldsm_x2(pp_s + q * (NP * 512) + atc_poff(row, j0 + ((lane >> 3) & 1) * 8), pb0, pb1);
              mma_bf16_16816(pacc[q][u], va, pb0, pb1);
            }
          }
        }
      }
      if (gi == my_last) {  // this warp group's last P.V of the chunk: its V rows may be replaced
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_v);
      }
      // partial record of each live pair: acc[e] = (o0 + o1) + o2, then m and l
#pragma unroll
      for (int u = 0; u < NPT; ++u)
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int pl = u * 8 + 2 * t4 + cc;
          if (pl >= gp || !live_s[wg][pl]) continue;
          const int p = pg0 + pl;
          const int i = p / a.G, g = p % a.G;
          const int hq = hk * a.G + g;
          float* rec = a.part + (((size_t)(t0 + i - a.t_base) * a.Hq + hq) * a.max_chunks + c) * (128 + 4);
          const int e = wl * 16 + g8;
          rec[e] = (pacc[0][u][cc] + pacc[1][u][cc]) + pacc[2][u][cc];
          rec[e + 8] = (pacc[0][u][2 + cc] + pacc[1][u][2 + cc]) + pacc[2][u][2 + cc];
          if (wl == 0 && g8 == 0) {
            rec[128] = m_s[wg][pl];
            rec[129] = l_s[wg][pl];
          }
        }
      gsync();  // the next group overwrites q, S, the probability parts and the statistics
    }
    if (!v_ready) {  // a warp group with no pair group still takes part in the chunk's V set-up
      v_prepare();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_v);
    }
  }
  if (a.merge_in_cta) {
    csync();  // every chunk record of the CTA is written
    for (int p = warp; p < npairs; p += NCW) {
      const int t = t0 + p / a.G, hq = hk * a.G + p % a.G;
      const int nc = min(pos_s[t - t0] / a.chunk + 1, c_hi);
      merge_pair(a.part + ((size_t)(t - a.t_base) * a.Hq + hq) * a.max_chunks * (128 + 4), nc, 128, lane, a.out,
                 (size_t)t * a.Hq * 128 + hq * 128, 0);
    }
  }
}

// ---------------------------------------------------------------------------
// Decode schedule of the same computation (one query per block, G <= 8 q
// heads: one 8-pair tile).  attn_tc_kernel<1, RING> walks each chunk as
// scores -> softmax -> P.V, so at every chunk boundary the next chunk's keys
// are only requested while P.V of the current one drains the ring.  Here a
// CTA first streams the K rows of its whole segment (at most ATD_SEG chunks)
// and keeps every score in shared memory; then it runs the softmax of every
// (chunk, pair) of the segment, one warp each, while the first V rows arrive,
// keeping the probability parts of every chunk; then it streams the V rows
// through P.V without a pause at the chunk boundaries.  All eight warps score:
// warps 0-3 the even 64-key sub-tiles, warps 4-7 the odd ones.  Every score, every
// softmax and every P.V chain is the instruction sequence of attn_tc_kernel
// (each score one warp's chain of 8 ascending k16 mma over the head; the same
// softmax row function; the same 3-part P split and per-part
// chains over ascending 16-key steps; the same record and merge), so the two
// kernels, and prefill and decode, give the same bits.
constexpr int ATD_SEG = 3;                   // chunks per CTA (scores of all of them are kept)
constexpr int ATD_SST = ATD_SEG * 256 + 4;  // row stride of the score rows (floats)

// Shared memory of attn_dec_kernel<RING, NP>: NP pair rows of scores and of the
// probability parts of every chunk of the segment (NP = 4 when a kv head has at
// most 4 q heads, which leaves room for a deeper ring at two CTAs per SM).  With
// NP = 4 the chunk records of the segment also stay in shared memory when the
// CTA merges them itself (NP = 8 would then no longer fit two CTAs per SM).
__host__ __device__ constexpr bool atd_smem_records(int np) { return np <= 4; }
__host__ __device__ inline size_t atd_smem_bytes(int ring, int np) {
  return (size_t)ring * 16384            // K/V sub-tiles: [2 halves][64 keys][128 B]
         + 8 * 256                       // q tile: [2 halves][8 pairs][128 B]
         + (size_t)np * ATD_SST * 4      // scores [NP][ATD_SST]
         + (size_t)ATD_SEG * 3 * np * 512  // probability parts [chunk][3][NP][256 keys] bf16, swizzled
         + (atd_smem_records(np) ? (size_t)np * ATD_SEG * (128 + 4) * 4 : 0)  // chunk records [NP][chunk][132]
         + 1024;
}

template <int RING, int NP>
__global__ void __launch_bounds__(ATC_THREADS)
    attn_dec_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ AttnPlan plan, const AttnArgs a) {
  if (!a.pre_kv) {
    pdl_wait();
    pdl_trigger();
  }
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[RING];
  __shared__ __align__(8) uint64_t empty_bar[RING];
  __shared__ float m_s[ATD_SEG][NP], l_s[ATD_SEG][NP];
  __shared__ int live_s[ATD_SEG][NP];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int b = blockIdx.x, sg = blockIdx.y, hk = blockIdx.z;
  if (b >= plan.n) return;
  const int t0 = plan.blk[b].x;  // one query per block
  const int s = a.slot[t0];
  const int pmax = a.pos[t0];
  const int c_lo = sg * a.seg_len;
  int c_hi = min(pmax / a.chunk + 1, c_lo + a.seg_len);
  if (c_hi > a.max_chunks) {  // device position beyond what the launch was planned for
    if (threadIdx.x == 0) dev_flag(DEVERR_CAPACITY);
    c_hi = a.max_chunks;
  }
  if (c_lo >= c_hi) return;
  const int npairs = a.G;  // <= NP
  const int cache_base = ((s * a.n_layers + a.layer) * a.Hkv + hk) * a.cap;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  constexpr uint32_t SUB = 16384;
  constexpr int PPART = NP * 512;  // bytes of one probability part of one chunk
  uint8_t* qt = smem + RING * SUB;                            // [2][8][128 B]
  float* S = reinterpret_cast<float*>(qt + 8 * 256);          // [NP][ATD_SST]
  uint8_t* Pp = reinterpret_cast<uint8_t*>(S + NP * ATD_SST);  // [ATD_SEG][3][NP][512 B]
  const uint32_t qt_s = smem_u32(qt), pp_s = smem_u32(Pp);
  // chunk records: in shared memory when this CTA merges them (no round trip
  // through L2 between the last P.V and the merge), else in the workspace
  const bool rec_smem = atd_smem_records(NP) && a.merge_in_cta;
  float* recs = reinterpret_cast<float*>(Pp + ATD_SEG * 3 * NP * 512);  // [NP][ATD_SEG][132]
  auto nsub_of = [&](int c) { return (min(a.chunk, pmax - c * a.chunk + 1) + ATT_SUB - 1) / ATT_SUB; };

  if (tid == 0) {
    for (int r = 0; r < RING; ++r) {
      mbar_init(&full_bar[r], 1);
      mbar_init(&empty_bar[r], ATT_THREADS / 32);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == ATT_THREADS / 32) {
    // ---- producer warp, one lane: every K sub-tile of the segment, then every V sub-tile
    if (lane == 0) {
      const uint64_t kvpol = l2_evict_first();  // each cached row is read once per step
      // With pre_kv the first ring fill is requested before the dependency
      // wait: K sub-tiles whose keys all lie below the token's own row (the one
      // row the previous kernel writes), in stream order up to the first that
      // does not.
      int pre = 0;
      if (a.pre_kv) {
        for (int pc = c_lo; pc < c_hi && pre < RING; ++pc) {
          const int pns = nsub_of(pc);
          int st = 0;
          for (; st < pns && pre < RING && pc * a.chunk + (st + 1) * ATT_SUB <= pmax; ++st, ++pre) {
            mbar_arrive_expect_tx(&full_bar[pre], SUB);
            tma_load_3d_hint(smem + pre * SUB, &tmK, 0, cache_base + pc * a.chunk + st * ATT_SUB, 0, &full_bar[pre],
                             kvpol);
          }
          if (st < pns) break;
        }
        pdl_wait();
      }
      int lp = 0;
      for (int isv = 0; isv < 2; ++isv)
        for (int pc = c_lo; pc < c_hi; ++pc) {
          const int pns = nsub_of(pc);
          for (int st = 0; st < pns; ++st, ++lp) {
            if (lp < pre) continue;  // requested before the wait
            const int slot = lp % RING;
            if (lp >= RING && !mbar_wait(&empty_bar[slot], (uint32_t)(((lp / RING) - 1) & 1), SITE_ATTN_TC | 0x90))
              return;
            mbar_arrive_expect_tx(&full_bar[slot], SUB);
            tma_load_3d_hint(smem + slot * SUB, isv ? &tmV : &tmK, 0, cache_base + pc * a.chunk + st * ATT_SUB, 0,
                             &full_bar[slot], kvpol);
          }
        }
    }
    return;
  }

  int L = 0;
  auto consume_wait = [&]() {
    (void)mbar_wait(&full_bar[L % RING], (uint32_t)((L / RING) & 1), SITE_ATTN_TC | 0x100);
  };
  auto release = [&]() {
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[L % RING]);
    ++L;
  };
  auto cbar = []() { asm volatile("bar.sync 1, %0;" ::"n"(ATT_THREADS) : "memory"); };
  if (a.pre_kv) {  // q, and every output, depend on the previous kernel
    pdl_wait();
    pdl_trigger();
  }

  // q tile (bf16, 128-byte swizzle per half; rows past the group are zero) and the q^T fragments
  for (int idx = tid; idx < 8 * 16; idx += ATT_THREADS) {
    const int row = idx >> 4, ch = idx & 15;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (row < npairs)
      v = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.q) + (size_t)t0 * a.Hq * 128 +
                                          (hk * a.G + row) * 128 + ch * 8);
    const int half = ch >> 3, cc = ch & 7;
    *reinterpret_cast<uint4*>(qt + half * (8 * 128) + row * 128 + ((cc ^ (row & 7)) << 4)) = v;
  }
  cbar();
  const int kt = warp & 3, par = warp >> 2;  // 16-key slice of a sub-tile; sub-tile parity this warp scores
  uint32_t qb[8][2];
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const int row = lane & 7;
    const int half = kk >> 2, ch = 2 * (kk & 3) + ((lane >> 3) & 1);
    ldsm_x2(qt_s + half * (8 * 128) + row * 128 + ((ch ^ (row & 7)) << 4), qb[kk][0], qb[kk][1]);
  }

  // ---- phase 1: scores of every chunk of the segment, S[pair][(c - c_lo) * 256 + key]
  for (int c = c_lo; c < c_hi; ++c) {
    const int nsub = nsub_of(c);
    float* Sc = S + (c - c_lo) * 256;
    for (int st = 0; st < nsub; ++st) {
      consume_wait();
      if ((st & 1) == par) {
        const uint32_t kb = smem_u32(smem + (L % RING) * SUB);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int krow = kt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int half = kk >> 2, ch = 2 * (kk & 3) + (lane >> 4);
          uint32_t ka[4];
          ldsm_x4(kb + half * 8192 + krow * 128 + ((ch ^ (krow & 7)) << 4), ka[0], ka[1], ka[2], ka[3]);
          mma_bf16_16816(acc, ka, qb[kk][0], qb[kk][1]);
        }
        const int pr = 2 * t4;
        const int j = st * ATT_SUB + kt * 16 + g8;
        if (pr < NP) {
          Sc[pr * ATD_SST + j] = acc[0] * a.scale;
          Sc[pr * ATD_SST + j + 8] = acc[2] * a.scale;
        }
        if (pr + 1 < NP) {
          Sc[(pr + 1) * ATD_SST + j] = acc[1] * a.scale;
          Sc[(pr + 1) * ATD_SST + j + 8] = acc[3] * a.scale;
        }
      }
      release();
    }
  }
  cbar();  // every score is in S

  // ---- phase 2: the softmax of every (chunk, pair) of the segment, one warp each,
  // while the V sub-tiles stream into the ring
  const int nch = c_hi - c_lo;
  for (int task = warp; task < nch * npairs; task += ATT_THREADS / 32) {
    const int cl = task / npairs, pl = task % npairs;
    const int key0 = (c_lo + cl) * a.chunk;
    const int nvalid = min(a.chunk, pmax - key0 + 1);
    const int lim = pmax - key0;  // keys j <= lim are visible to the query
    float mx, sum;
    atc_softmax_row(S + cl * 256 + pl * ATD_SST, Pp + cl * (3 * PPART), PPART, pl, lim, nvalid, lane, mx, sum);
    if (lane == 0) {
      m_s[cl][pl] = mx;
      l_s[cl][pl] = sum;
      live_s[cl][pl] = lim >= 0;
    }
  }
  cbar();

  // ---- phase 3: P.V of every chunk, the V stream without pauses.  Warp w owns
  // head elements 16w..16w+15 (one m16 tile of V^T); pair rows past NP read a
  // real row (their columns of the product are never stored).
  for (int c = c_lo; c < c_hi; ++c) {
    const int cl = c - c_lo;
    const int nvalid = min(a.chunk, pmax - c * a.chunk + 1);
    const int nsub = (nvalid + ATT_SUB - 1) / ATT_SUB;
    const uint32_t pc_s = pp_s + cl * (3 * PPART);
    float pacc[3][4];
#pragma unroll
    for (int q = 0; q < 3; ++q) pacc[q][0] = pacc[q][1] = pacc[q][2] = pacc[q][3] = 0.f;
    for (int st = 0; st < nsub; ++st) {
      consume_wait();
      uint8_t* vbuf = smem + (L % RING) * SUB;
      const int vrows = nvalid - st * ATT_SUB;
      if (vrows < ATT_SUB) {  // zero the rows past the last valid key
        for (int idx = tid; idx < (ATT_SUB - vrows) * 16; idx += ATT_THREADS) {
          const int r = vrows + (idx >> 4), ch = idx & 15;
          *reinterpret_cast<uint4*>(vbuf + (ch >> 3) * 8192 + r * 128 + ((ch & 7) << 4)) = make_uint4(0u, 0u, 0u, 0u);
        }
        cbar();
      }
      const uint32_t vb = smem_u32(vbuf);
      const int nk16 = min(4, (vrows + 15) / 16);
      for (int kk = 0; kk < nk16; ++kk) {
        uint32_t va[4];
        {
          const int krow = kk * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
          const int e0 = warp * 16 + ((lane >> 3) & 1) * 8;
          const int half = e0 >> 6, ch = (e0 & 63) >> 3;
          ldsm_x4_trans(vb + half * 8192 + krow * 128 + ((ch ^ (krow & 7)) << 4), va[0], va[1], va[2], va[3]);
        }
        const int j0 = st * ATT_SUB + kk * 16;
#pragma unroll
        for (int q = 0; q < 3; ++q) {
          uint32_t pb0, pb1;
          const int row = (lane & 7) % NP;
          ldsm_x2(pc_s + q * PPART + atc_poff(row, j0 + ((lane >> 3) & 1) * 8), pb0, pb1);
          mma_bf16_16816(pacc[q], va, pb0, pb1);
        }
      }
      release();
    }
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      const int pl = 2 * t4 + cc;
      if (pl >= npairs || !live_s[cl][pl]) continue;
      const int hq = hk * a.G + pl;
      float* rec = rec_smem ? recs + ((size_t)pl * ATD_SEG + (c - c_lo)) * (128 + 4)
                            : a.part + (((size_t)(t0 - a.t_base) * a.Hq + hq) * a.max_chunks + c) * (128 + 4);
      const int e = warp * 16 + g8;
      rec[e] = (pacc[0][cc] + pacc[1][cc]) + pacc[2][cc];
      rec[e + 8] = (pacc[0][2 + cc] + pacc[1][2 + cc]) + pacc[2][2 + cc];
      if (warp == 0 && g8 == 0) {
        rec[128] = m_s[cl][pl];
        rec[129] = l_s[cl][pl];
      }
    }
  }
  if (a.merge_in_cta) {
    cbar();  // every chunk record of the CTA is written
    for (int p = warp; p < npairs; p += ATT_THREADS / 32) {
      const int hq = hk * a.G + p;
      const int nc = min(pmax / a.chunk + 1, c_hi);
      merge_pair(rec_smem ? recs + (size_t)p * ATD_SEG * (128 + 4)
                          : a.part + ((size_t)(t0 - a.t_base) * a.Hq + hq) * a.max_chunks * (128 + 4),
                 nc, 128, lane, a.out, (size_t)t0 * a.Hq * 128 + hq * 128, 0);
    }
  }
}

// One warp per (token, q head): fixed ascending merge of the chunk partials.
__global__ void attn_merge_kernel(const float* __restrict__ part, const int32_t* __restrict__ pos, void* __restrict__ out,
                                  int t_base, int T, int Hq, int d, int chunk, int max_chunks, int f32) {
  pdl_wait();
  pdl_trigger();
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= T * Hq) return;
  const int tl = gw / Hq, hq = gw % Hq;
  const int t = t_base + tl;
  int nc = pos[t] / chunk + 1;
  if (nc > max_chunks) {  // device position beyond what the launch was planned for: never read past the partials
    if (lane == 0) dev_flag(DEVERR_CAPACITY);
    nc = max_chunks;
  }
  merge_pair(part + ((size_t)tl * Hq + hq) * max_chunks * (d + 4), nc, d, lane, out, (size_t)t * Hq * d + hq * d, f32);
}

}  // namespace bi
