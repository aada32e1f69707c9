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
//   * chunk numerator acc[e] = sum_j p_j v_j[e]: sequential FMA over the valid
//     keys in ascending order (keys past the query add exact zeros, so it is
//     the same sum whether later queries share the tile or not);
//   * merge over chunks 0..pos/CH: M = max m_c, L = sum_c l_c exp(m_c - M),
//     o = sum_c acc_c exp(m_c - M), all in ascending chunk order; out = o / L.
// A query's result depends only on its q and the cache rows 0..pos it reads.
#pragma once
#include "common.cuh"

namespace bi {

constexpr int ATT_THREADS = 256;
constexpr int ATT_CHUNK = BI_ATTN_CHUNK;  // 256
constexpr int ATT_MAX_PAIRS = 32;         // (query, q-head) pairs per CTA
constexpr int ATT_MAX_BLOCKS = 1024;      // query blocks per launch
constexpr int ATT_TOKEN_GROUP = 1024;     // tokens per partials workspace pass

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
};

__host__ __device__ inline int att_ninner(int d, int f32) { return d * (f32 ? 4 : 2) / 128; }

// Grid: (block, chunk, kv head).  Dynamic smem: K tile, V tile (the same
// buffer in f32 mode), q pairs (fp32), scores/probabilities [pairs][CH].
__global__ void __launch_bounds__(ATT_THREADS)
    attn_partial_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ AttnPlan plan, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar[2];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int b = blockIdx.x, c = blockIdx.y, hk = blockIdx.z;
  if (b >= plan.n) return;
  const int t0 = plan.blk[b].x, nq = plan.blk[b].y;
  const int s = a.slot[t0];
  const int pmax = a.pos[t0 + nq - 1];
  const int key0 = c * a.chunk;
  if (key0 > pmax) return;  // chunk beyond every query of the block
  const int nvalid = min(a.chunk, pmax - key0 + 1);
  const int nsub = (nvalid + 63) / 64;
  const int ninner = att_ninner(a.d, a.f32);
  const int esz = a.f32 ? 4 : 2;
  const int boxe = 128 / esz;
  const size_t kv_region = (size_t)ATT_CHUNK * a.d * esz;
  uint8_t* kbuf = smem;
  uint8_t* vbuf = a.f32 ? smem : smem + kv_region;
  float* qs = reinterpret_cast<float*>(smem + (a.f32 ? kv_region : 2 * kv_region));
  float* S = qs + ATT_MAX_PAIRS * a.d;
  const int npairs = nq * a.G;
  const int row_base = ((s * a.n_layers + a.layer) * a.Hkv + hk) * a.cap + key0;
  const uint32_t bytes = nsub * ninner * 64 * 128;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_expect_tx(&bar[0], bytes);
    for (int sb = 0; sb < nsub; ++sb)
      for (int ib = 0; ib < ninner; ++ib)
        tma_load_2d(kbuf + ib * (ATT_CHUNK * 128) + sb * 64 * 128, &tmK, ib * boxe, row_base + sb * 64, &bar[0]);
    if (!a.f32) {
      mbar_arrive_expect_tx(&bar[1], bytes);
      for (int sb = 0; sb < nsub; ++sb)
        for (int ib = 0; ib < ninner; ++ib)
          tma_load_2d(vbuf + ib * (ATT_CHUNK * 128) + sb * 64 * 128, &tmV, ib * boxe, row_base + sb * 64, &bar[1]);
    }
  }
  // q of the block's (query, head) pairs -> fp32 smem; pair p = i*G + g, head hk*G + g
  for (int idx = tid; idx < npairs * a.d; idx += ATT_THREADS) {
    const int p = idx / a.d, e = idx % a.d;
    const int i = p / a.G, g = p % a.G;
    const int hq = hk * a.G + g;
    qs[p * a.d + e] = load_act(a.q, (size_t)(t0 + i) * a.Hq * a.d + hq * a.d + e, a.f32);
  }
  __syncthreads();
  if (!mbar_wait(&bar[0], 0)) return;

  // ---- scores: thread j = key j of the chunk
  {
    const int j = tid;
    if (j < nvalid) {
      float acc[ATT_MAX_PAIRS];
#pragma unroll
      for (int p = 0; p < ATT_MAX_PAIRS; ++p) acc[p] = 0.f;
      const int nch = a.d * esz / 16;  // 16-byte chunks per key row
      for (int ch = 0; ch < nch; ++ch) {
        const int ib = ch >> 3, cc = ch & 7;
        const uint8_t* rowp = kbuf + ib * (ATT_CHUNK * 128) + j * 128;
        const uint4 u = *reinterpret_cast<const uint4*>(rowp + ((cc ^ (j & 7)) << 4));
        float kv[8];
        int ne;
        if (a.f32) {
          kv[0] = __uint_as_float(u.x); kv[1] = __uint_as_float(u.y);
          kv[2] = __uint_as_float(u.z); kv[3] = __uint_as_float(u.w);
          ne = 4;
        } else {
          kv[0] = bf16lo(u.x); kv[1] = bf16hi(u.x); kv[2] = bf16lo(u.y); kv[3] = bf16hi(u.y);
          kv[4] = bf16lo(u.z); kv[5] = bf16hi(u.z); kv[6] = bf16lo(u.w); kv[7] = bf16hi(u.w);
          ne = 8;
        }
        const int e0 = ch * ne;
#pragma unroll
        for (int p = 0; p < ATT_MAX_PAIRS; ++p) {
          if (p < npairs) {
            const float* qp = qs + p * a.d + e0;
            if (ne == 8) {
              const float4 q0 = *reinterpret_cast<const float4*>(qp);
              const float4 q1 = *reinterpret_cast<const float4*>(qp + 4);
              float x = acc[p];
              x = fmaf(q0.x, kv[0], x); x = fmaf(q0.y, kv[1], x); x = fmaf(q0.z, kv[2], x); x = fmaf(q0.w, kv[3], x);
              x = fmaf(q1.x, kv[4], x); x = fmaf(q1.y, kv[5], x); x = fmaf(q1.z, kv[6], x); x = fmaf(q1.w, kv[7], x);
              acc[p] = x;
            } else {
              const float4 q0 = *reinterpret_cast<const float4*>(qp);
              float x = acc[p];
              x = fmaf(q0.x, kv[0], x); x = fmaf(q0.y, kv[1], x); x = fmaf(q0.z, kv[2], x); x = fmaf(q0.w, kv[3], x);
              acc[p] = x;
            }
          }
        }
      }
#pragma unroll
      for (int p = 0; p < ATT_MAX_PAIRS; ++p)
        if (p < npairs) S[p * ATT_CHUNK + j] = acc[p] * a.scale;
    }
  }
  __syncthreads();
  if (a.f32 && tid == 0) {  // f32: V reuses the K buffer, load it now
    mbar_arrive_expect_tx(&bar[1], bytes);
    for (int sb = 0; sb < nsub; ++sb)
      for (int ib = 0; ib < ninner; ++ib)
        tma_load_2d(vbuf + ib * (ATT_CHUNK * 128) + sb * 64 * 128, &tmV, ib * boxe, row_base + sb * 64, &bar[1]);
  }

  // ---- softmax per pair: warp w handles pairs w, w+8, ...; lane i keys i + 32k
  __shared__ float m_s[ATT_MAX_PAIRS], l_s[ATT_MAX_PAIRS];
  __shared__ int live_s[ATT_MAX_PAIRS];
  for (int p = warp; p < npairs; p += ATT_THREADS / 32) {
    const int i = p / a.G;
    const int lim = a.pos[t0 + i] - key0;  // keys j <= lim are visible to this query
    float mx = -INFINITY;
#pragma unroll
    for (int k = 0; k < ATT_CHUNK / 32; ++k) {
      const int j = lane + 32 * k;
      if (j <= lim && j < nvalid) mx = fmaxf(mx, S[p * ATT_CHUNK + j]);
    }
    mx = warp_max(mx);
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < ATT_CHUNK / 32; ++k) {
      const int j = lane + 32 * k;
      float pj = 0.f;
      if (j <= lim && j < nvalid) pj = expf(S[p * ATT_CHUNK + j] - mx);
      if (j < nvalid) S[p * ATT_CHUNK + j] = pj;
      sum += pj;
    }
    sum = warp_sum_fixed(sum);
    if (lane == 0) {
      m_s[p] = mx;
      l_s[p] = sum;
      live_s[p] = lim >= 0;
    }
  }
  __syncthreads();
  if (!mbar_wait(&bar[1], 0)) return;

  // ---- PV: thread -> (e = tid % d, pairs p = tid / d + k * (256 / d))
  {
    const int e = tid % a.d;
    const int pstep = ATT_THREADS / a.d;
    const int p0 = tid / a.d;
    const int ib = (e * esz) >> 7;            // inner box of element e
    const int cc = ((e * esz) & 127) >> 4;    // 16-byte chunk within the 128-byte row
    const int within = (e * esz) & 15;
    float acc[ATT_MAX_PAIRS / 2];
#pragma unroll
    for (int k = 0; k < ATT_MAX_PAIRS / 2; ++k) acc[k] = 0.f;
    const uint8_t* vb = vbuf + ib * (ATT_CHUNK * 128) + within;
    for (int j = 0; j < nvalid; ++j) {
      const uint8_t* vp = vb + j * 128 + ((cc ^ (j & 7)) << 4);
      const float v = a.f32 ? *reinterpret_cast<const float*>(vp) : bf16_bits_to_f32(*reinterpret_cast<const uint16_t*>(vp));
#pragma unroll
      for (int k = 0; k < ATT_MAX_PAIRS / 2; ++k) {
        const int p = p0 + k * pstep;
        if (p < npairs) acc[k] = fmaf(S[p * ATT_CHUNK + j], v, acc[k]);
      }
    }
#pragma unroll
    for (int k = 0; k < ATT_MAX_PAIRS / 2; ++k) {
      const int p = p0 + k * pstep;
      if (p < npairs && live_s[p]) {
        const int i = p / a.G, g = p % a.G;
        const int hq = hk * a.G + g;
        float* rec = a.part + (((size_t)(t0 + i - a.t_base) * a.Hq + hq) * a.max_chunks + c) * (a.d + 4);
        rec[e] = acc[k];
        if (e == 0) {
          rec[a.d] = m_s[p];
          rec[a.d + 1] = l_s[p];
        }
      }
    }
  }
}

// One warp per (token, q head): fixed ascending merge of the chunk partials.
__global__ void attn_merge_kernel(const float* __restrict__ part, const int32_t* __restrict__ pos, void* __restrict__ out,
                                  int t_base, int T, int Hq, int d, int chunk, int max_chunks, int f32) {
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
  const float* base = part + ((size_t)tl * Hq + hq) * max_chunks * (d + 4);
  float M = -INFINITY;
  for (int c = 0; c < nc; ++c) M = fmaxf(M, base[(size_t)c * (d + 4) + d]);
  float L = 0.f;
  float o[4] = {0.f, 0.f, 0.f, 0.f};
  const int ne = d / 32;
  for (int c = 0; c < nc; ++c) {
    const float* rec = base + (size_t)c * (d + 4);
    const float w = expf(rec[d] - M);
    L = fmaf(rec[d + 1], w, L);
    for (int k = 0; k < ne; ++k) o[k] = fmaf(rec[lane + 32 * k], w, o[k]);
  }
  for (int k = 0; k < ne; ++k) store_act(out, (size_t)t * Hq * d + hq * d + lane + 32 * k, o[k] / L, f32);
}

}  // namespace bi
