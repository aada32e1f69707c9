// bi_lmhead_logprob kernels: vocabulary-chunk partials, fixed-order merge,
// and the selective FP32 recompute bookkeeping.
//
// ("Meituan bitwise train/infer consistency": logprob accumulation is one of
// the reductions whose order is fixed; "Greedy Decoding Is Not
// Precision-Invariant", method section: top-two logit margin, FP32 LM-head
// recompute only when it falls below a threshold.)
//
// Per row and per chunk of BI_VOCAB_CHUNK = 256 logits, one warp (lane l holds
// logits l, l + 32, ..., l + 224 of the chunk): max (exact), sum exp(z - max)
// with a fixed tree (each lane's 8 terms in ascending order, then an xor
// butterfly), top-1 and top-2 as (value, id) under the total order "larger
// value, then lower id" (exact, order-free), and the target logit if the
// target falls in the chunk.
// Merge per row: M = max over chunks (exact); S = sum_c s_c exp(m_c - M):
//   lane i of one warp sums chunks i, i+32, ... in ascending order, then a
//   fixed xor-butterfly; lse = M + ln S; top-2 merged exactly.
#pragma once
#include "common.cuh"

namespace bi {

constexpr int LM_CHUNK = BI_VOCAB_CHUNK;  // 256
struct LmPart {
  float mx, sum, v1, v2, zt;
  int i1, i2, has_t;
};

// (v, i) beats (w, j) if v > w, or v == w and i < j.
__device__ __forceinline__ bool lm_better(float v, int i, float w, int j) { return v > w || (v == w && i < j); }
__device__ __forceinline__ void lm_top2_insert(float& v1, int& i1, float& v2, int& i2, float v, int i) {
  if (lm_better(v, i, v1, i1)) {
    v2 = v1; i2 = i1; v1 = v; i1 = i;
  } else if (lm_better(v, i, v2, i2)) {
    v2 = v; i2 = i;
  }
}
__device__ __forceinline__ void lm_top2_warp(float& v1, int& i1, float& v2, int& i2) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov1 = __shfl_xor_sync(0xffffffffu, v1, o), ov2 = __shfl_xor_sync(0xffffffffu, v2, o);
    const int oi1 = __shfl_xor_sync(0xffffffffu, i1, o), oi2 = __shfl_xor_sync(0xffffffffu, i2, o);
    lm_top2_insert(v1, i1, v2, i2, ov1, oi1);
    lm_top2_insert(v1, i1, v2, i2, ov2, oi2);
  }
}

// Grid (ceil(n_chunks / LM_CPB), B), LM_CPB warps per CTA, warp w taking
// chunk blockIdx.x * LM_CPB + w of grid row blockIdx.y.  logits: [rows][ldz]
// f32.  Row r of the grid is logits row r; rows >= *count (when count !=
// nullptr) are skipped.  target: per-row target id (nullptr: none); rows_map
// maps grid row -> target row (nullptr: identity).
// parts == 3: the logit is (z0 + z1) + z2, the three partial products of the
// exact bf16 split of an f32 hidden row (layouts below).
constexpr int LM_CPB = 8;  // vocabulary chunks (warps) per CTA

__global__ void __launch_bounds__(32 * LM_CPB)
    lm_partial_kernel(const float* __restrict__ logits, size_t ldz, int V, const int32_t* __restrict__ target,
                      const int32_t* __restrict__ rows_map, const int* __restrict__ count, LmPart* __restrict__ part,
                      int n_chunks, int parts, int pstride, const float* __restrict__ parts_z) {
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.y;
  if (count && r >= *count) return;
  const int lane = threadIdx.x & 31;
  const int c = blockIdx.x * LM_CPB + (threadIdx.x >> 5);
  if (c >= n_chunks) return;
  constexpr int PER = LM_CHUNK / 32;
  float z[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int v = c * LM_CHUNK + lane + 32 * j;
    float zv = -INFINITY;
    if (v < V) {
      if (parts == 3) {  // row r of the compacted list: (z0 + z1) + z2 of its row src
        // z0 = logits row src (the main pass on p0 = bf16(h)); z1, z2 at rows
        // src + pstride, src + 2 pstride of logits (one-pass layout, pstride > 0)
        // or at rows 2r, 2r + 1 of parts (second pass, pstride == 0)
        const size_t src = rows_map[r];
        const float z0 = logits[src * ldz + v];
        if (pstride > 0)
          zv = (z0 + logits[(src + pstride) * ldz + v]) + logits[(src + 2 * pstride) * ldz + v];
        else
          zv = (z0 + parts_z[(size_t)(2 * r) * ldz + v]) + parts_z[(size_t)(2 * r + 1) * ldz + v];
      } else {
        zv = logits[(size_t)r * ldz + v];
      }
    }
    z[j] = zv;
  }
  float mx = z[0];
#pragma unroll
  for (int j = 1; j < PER; ++j) mx = fmaxf(mx, z[j]);
  const float M = warp_max(mx);
  float v1 = -INFINITY, v2 = -INFINITY;
  int i1 = 0x7fffffff, i2 = 0x7fffffff;
  float e = 0.f, zt = 0.f;
  int has = 0;
  const int tg = target ? target[rows_map ? rows_map[r] : r] : -1;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int v = c * LM_CHUNK + lane + 32 * j;
    if (v < V) {
      lm_top2_insert(v1, i1, v2, i2, z[j], v);
      e += expf(z[j] - M);
      if (v == tg) {
        zt = z[j];
        has = 1;
      }
    }
  }
  const float S = warp_sum_fixed(e);
  lm_top2_warp(v1, i1, v2, i2);
  const unsigned hb = __ballot_sync(0xffffffffu, has);
  zt = __shfl_sync(0xffffffffu, zt, hb ? __ffs(hb) - 1 : 0);
  if (lane == 0) {
    LmPart pr;
    pr.mx = M; pr.sum = S; pr.v1 = v1; pr.i1 = i1; pr.v2 = v2; pr.i2 = i2;
    pr.has_t = hb != 0; pr.zt = hb ? zt : 0.f;
    part[(size_t)r * n_chunks + c] = pr;
  }
}

// One warp per row.  mode_recompute = 0: main pass (writes every output and
// sets the flag); 1: recompute pass (rows given by rows_map, writes lse,
// logprob, argmax and recomputed = 1; margin keeps the main-pass value).
__global__ void lm_merge_kernel(const LmPart* __restrict__ part, int n_chunks, int B, const int* __restrict__ count,
                                const int32_t* __restrict__ rows_map, const int32_t* __restrict__ target,
                                float thresh, int mode_recompute, float* __restrict__ logprob, float* __restrict__ lse,
                                int32_t* __restrict__ argmax, float* __restrict__ margin,
                                uint8_t* __restrict__ recomputed, uint8_t* __restrict__ flag) {
  pdl_wait();
  pdl_trigger();
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int nrows = count ? min(B, *count) : B;
  if (r >= nrows) return;
  const LmPart* pr = part + (size_t)r * n_chunks;
  float M = -INFINITY;
  for (int c = lane; c < n_chunks; c += 32) M = fmaxf(M, pr[c].mx);
  M = warp_max(M);
  float S = 0.f, zt = 0.f;
  int has = 0;
  float v1 = -INFINITY, v2 = -INFINITY;
  int i1 = 0x7fffffff, i2 = 0x7fffffff;
  for (int c = lane; c < n_chunks; c += 32) {
    const LmPart q = pr[c];
    S = fmaf(q.sum, expf(q.mx - M), S);
    lm_top2_insert(v1, i1, v2, i2, q.v1, q.i1);
    lm_top2_insert(v1, i1, v2, i2, q.v2, q.i2);
    if (q.has_t) {
      has = 1;
      zt = q.zt;
    }
  }
  S = warp_sum_fixed(S);
  lm_top2_warp(v1, i1, v2, i2);
  const unsigned hb = __ballot_sync(0xffffffffu, has);
  const int src = hb ? __ffs(hb) - 1 : 0;
  zt = __shfl_sync(0xffffffffu, zt, src);
  if (lane != 0) return;
  const float L = M + logf(S);
  const int orow = rows_map ? rows_map[r] : r;
  const int tg = target ? target[orow] : -1;
  const float lp = (tg >= 0 && hb) ? zt - L : v1 - L;
  lse[orow] = L;
  logprob[orow] = lp;
  argmax[orow] = i1;
  if (!mode_recompute) {
    const float mg = v1 - v2;
    margin[orow] = mg;
    const bool f = thresh > 0.f && mg < thresh;
    if (flag) flag[orow] = f;
    recomputed[orow] = 0;
  } else {
    recomputed[orow] = 1;
  }
}

// Ascending compaction of the flagged rows: list[k] = k-th flagged row.  CTA
// b handles row b: its rank is the number of flagged rows before it; CTA 0
// also writes the count.  With hc2 != nullptr (second-pass recompute) the
// row's f32 h is also split exactly into three bf16 parts (see
// lm_split_kernel); p1 and p2 are stored as rows 2k, 2k+1 of hc2 (the logits
// of p0 = bf16(h) are the main pass's).
__global__ void lm_compact_kernel(const uint8_t* __restrict__ flag, int B, const float* __restrict__ h, int H,
                                  int32_t* __restrict__ list, int* __restrict__ count, uint16_t* __restrict__ hc2) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x;
  __shared__ int rank_s;
  if (threadIdx.x < 32) {
    int before = 0, total = 0;
    for (int i = threadIdx.x; i < B; i += 32) {
      const int f = flag[i] != 0;
      before += (i < b) ? f : 0;
      total += f;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      before += __shfl_xor_sync(0xffffffffu, before, o);
      total += __shfl_xor_sync(0xffffffffu, total, o);
    }
    if (threadIdx.x == 0) {
      rank_s = before;
      if (b == 0) *count = total;
      if (flag[b]) list[before] = b;
    }
  }
  __syncthreads();
  if (!hc2 || !flag[b]) return;
  const int k = rank_s;
  for (int i = threadIdx.x; i < H; i += blockDim.x) {
    const float v = h[(size_t)b * H + i];
    const uint16_t p0 = f32_to_bf16_bits(v);
    const float r0 = v - bf16_bits_to_f32(p0);  // exact
    const uint16_t p1 = f32_to_bf16_bits(r0);
    const float r1 = r0 - bf16_bits_to_f32(p1);  // exact, at most 8 significant bits
    hc2[(size_t)(2 * k) * H + i] = p1;
    hc2[(size_t)(2 * k + 1) * H + i] = f32_to_bf16_bits(r1);
  }
}

// LM-head GEMM input.  parts == 1: row r of out is bf16(h_r) (round to nearest
// even).  parts == 3: h is also split exactly into three bf16 parts
// h = p0 + p1 + p2 (p0 = bf16(h), p1 = bf16(h - p0), p2 = h - p0 - p1; 8 + 8 + 8
// significant bits cover the 24 of an f32), stored as rows r, B + r and
// 2B + r, so one GEMM pass over W yields both the bf16-path logits (rows
// 0..B-1) and the parts of the FP32 logits of every row.
__global__ void lm_split_kernel(const float* __restrict__ h, uint16_t* __restrict__ out, size_t n, int parts) {
  pdl_wait();
  pdl_trigger();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const float v = h[i];
    const uint16_t p0 = f32_to_bf16_bits(v);
    out[i] = p0;
    if (parts == 3) {
      const float r0 = v - bf16_bits_to_f32(p0);  // exact
      const uint16_t p1 = f32_to_bf16_bits(r0);
      const float r1 = r0 - bf16_bits_to_f32(p1);  // exact, at most 8 significant bits
      out[n + i] = p1;
      out[2 * n + i] = f32_to_bf16_bits(r1);
    }
  }
}

}  // namespace bi
