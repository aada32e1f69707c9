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
struct __align__(16) LmPart {  // 32 bytes: read as two 16-byte halves by the merge
  float mx, sum, v1, v2, zt;
  int i1, i2, has_t;
};
static_assert(sizeof(LmPart) == 32, "LmPart layout");

__device__ __forceinline__ int warp_min_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
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

// Grid (ceil(n_chunks / LM_CPB), rows), LM_CPB warps per CTA, warp w taking
// chunk blockIdx.x * LM_CPB + w of grid row blockIdx.y.  logits: [rows][ldz]
// f32.  Grid rows >= *count (when count != nullptr) are skipped.  target:
// per-row target id (nullptr: none).  What grid row r computes:
//   parts 1: the logits of row r (rows_map, if given, maps r -> target row);
//   parts 3: the exact logits (z0 + z1) + z2 of the f32 hidden row src =
//     rows_map[r] (compacted flagged rows): z0 at row src of logits, z1 and z2
//     at rows src + pstride and src + 2 pstride (one-pass layout, pstride > 0)
//     or at rows 2r, 2r + 1 of parts_z (second pass, pstride == 0);
//   parts 4 (one-pass layout, every row both ways): rows r < pstride as parts
//     1, rows r >= pstride the exact logits of row src = r - pstride.
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
  const bool exact = parts == 3 || (parts == 4 && r >= pstride);
  // the hidden row this grid row belongs to (its target)
  const int src = parts == 4 ? (exact ? r - pstride : r) : (rows_map ? rows_map[r] : r);
  float z[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int v = c * LM_CHUNK + lane + 32 * j;
    float zv = -INFINITY;
    if (v < V) {
      if (!exact) {
        zv = logits[(size_t)r * ldz + v];
      } else {
        const float z0 = logits[(size_t)src * ldz + v];
        if (pstride > 0)
          zv = (z0 + logits[((size_t)src + pstride) * ldz + v]) + logits[((size_t)src + 2 * pstride) * ldz + v];
        else
          zv = (z0 + parts_z[(size_t)(2 * r) * ldz + v]) + parts_z[(size_t)(2 * r + 1) * ldz + v];
      }
    }
    z[j] = zv;
  }
  float mx = z[0];
#pragma unroll
  for (int j = 1; j < PER; ++j) mx = fmaxf(mx, z[j]);
  const float M = warp_max(mx);
  const int v0 = c * LM_CHUNK + lane;  // id of z[0]; z[j] has id v0 + 32 j
  float e = 0.f, zt = 0.f;
  int has = 0;
  const int tg = target ? target[src] : -1;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    if (v0 + 32 * j < V) {
      e += expf(z[j] - M);
      if (v0 + 32 * j == tg) {
        zt = z[j];
        has = 1;
      }
    }
  }
  const float S = warp_sum_fixed(e);
  // Top two (value, id) under "larger value, then lower id", from the exact
  // max: the first is the lowest valid id whose logit equals M, the second the
  // same rule over the chunk without the first.  Each stored value is the
  // owner lane's logit itself (so a -0 stays -0).  Rows of exact logits need
  // only the first: their margin is the main pass's.
  auto owner_value = [&](int id) {
    const int k = id - c * LM_CHUNK;  // 0..255, or out of range for "none"
    float mine = -INFINITY;
#pragma unroll
    for (int j = 0; j < PER; ++j)
      if (lane + 32 * j == k) mine = z[j];
    return __shfl_sync(0xffffffffu, mine, k & 31);
  };
  int c1 = 0x7fffffff;
#pragma unroll
  for (int j = PER - 1; j >= 0; --j)
    if (v0 + 32 * j < V && z[j] == M) c1 = v0 + 32 * j;
  const int i1 = warp_min_int(c1);
  const float v1 = i1 == 0x7fffffff ? -INFINITY : owner_value(i1);
  float v2 = -INFINITY;
  int i2 = 0x7fffffff;
  if (!exact) {
    float m2 = -INFINITY;
#pragma unroll
    for (int j = 0; j < PER; ++j)
      if (v0 + 32 * j < V && v0 + 32 * j != i1) m2 = fmaxf(m2, z[j]);
    const float M2 = warp_max(m2);
    int c2 = 0x7fffffff;
#pragma unroll
    for (int j = PER - 1; j >= 0; --j)
      if (v0 + 32 * j < V && v0 + 32 * j != i1 && z[j] == M2) c2 = v0 + 32 * j;
    i2 = warp_min_int(c2);
    if (i2 != 0x7fffffff) v2 = owner_value(i2);
  }
  const unsigned hb = __ballot_sync(0xffffffffu, has);
  zt = __shfl_sync(0xffffffffu, zt, hb ? __ffs(hb) - 1 : 0);
  if (lane == 0) {
    LmPart pr;
    pr.mx = M; pr.sum = S; pr.v1 = v1; pr.i1 = i1; pr.v2 = v2; pr.i2 = i2;
    pr.has_t = hb != 0; pr.zt = hb ? zt : 0.f;
    part[(size_t)r * n_chunks + c] = pr;
  }
}

// Merge of one row's chunk partials (one warp; every lane returns the results).
struct LmRow {
  float L, v1, v2, zt;
  int i1, has;
};
// Up to LM_MERGE_REG chunks per lane (n_chunks <= 32 * LM_MERGE_REG, vocabularies
// up to 163840) are read in one pass, every load issued at once: max, top-2 and
// the target need no order, and each chunk's (max, sum) stays in registers for
// the ordered sum.  Larger vocabularies take two passes over the partials.
// Either way lane l sums chunks l, l + 32, ... in ascending order.
constexpr int LM_MERGE_REG = 20;
__device__ __forceinline__ LmRow lm_merge_row(const LmPart* __restrict__ pr, int n_chunks, int lane) {
  float M = -INFINITY, S = 0.f, zt = 0.f;
  int has = 0;
  float v1 = -INFINITY, v2 = -INFINITY;
  int i1 = 0x7fffffff, i2 = 0x7fffffff;
  auto take = [&](const LmPart& q) {
    lm_top2_insert(v1, i1, v2, i2, q.v1, q.i1);
    lm_top2_insert(v1, i1, v2, i2, q.v2, q.i2);
    if (q.has_t) {
      has = 1;
      zt = q.zt;
    }
  };
  if (n_chunks <= 32 * LM_MERGE_REG) {
    float mxs[LM_MERGE_REG], sums[LM_MERGE_REG];
    constexpr int BATCH = LM_MERGE_REG / 2;  // partials loaded per batch, all before any is used
#pragma unroll
    for (int k0 = 0; k0 < LM_MERGE_REG; k0 += BATCH) {
      uint4 lo[BATCH], hi[BATCH];
#pragma unroll
      for (int k = 0; k < BATCH; ++k) {
        const int c = min(lane + 32 * (k0 + k), n_chunks - 1);  // in bounds; unused past n_chunks
        const uint4* q = reinterpret_cast<const uint4*>(pr + c);
        lo[k] = q[0];
        hi[k] = q[1];
      }
#pragma unroll
      for (int k = 0; k < BATCH; ++k) {
        LmPart q;
        q.mx = __uint_as_float(lo[k].x); q.sum = __uint_as_float(lo[k].y);
        q.v1 = __uint_as_float(lo[k].z); q.v2 = __uint_as_float(lo[k].w);
        q.zt = __uint_as_float(hi[k].x); q.i1 = (int)hi[k].y; q.i2 = (int)hi[k].z; q.has_t = (int)hi[k].w;
        const bool ok = lane + 32 * (k0 + k) < n_chunks;
        mxs[k0 + k] = ok ? q.mx : -INFINITY;
        sums[k0 + k] = ok ? q.sum : 0.f;
        if (ok) {
          M = fmaxf(M, q.mx);
          take(q);
        }
      }
    }
    M = warp_max(M);
#pragma unroll
    for (int k = 0; k < LM_MERGE_REG; ++k)
      if (lane + 32 * k < n_chunks) S = fmaf(sums[k], expf(mxs[k] - M), S);
  } else {
    for (int c = lane; c < n_chunks; c += 32) M = fmaxf(M, pr[c].mx);
    M = warp_max(M);
    for (int c = lane; c < n_chunks; c += 32) {
      const LmPart q = pr[c];
      S = fmaf(q.sum, expf(q.mx - M), S);
      take(q);
    }
  }
  S = warp_sum_fixed(S);
  lm_top2_warp(v1, i1, v2, i2);
  const unsigned hb = __ballot_sync(0xffffffffu, has);
  const int src = hb ? __ffs(hb) - 1 : 0;
  zt = __shfl_sync(0xffffffffu, zt, src);
  LmRow o;
  o.L = M + logf(S);
  o.v1 = v1;
  o.v2 = v2;
  o.i1 = i1;
  o.zt = zt;
  o.has = hb != 0;
  return o;
}

// One warp per row.  mode_recompute = 0: main pass (writes every output and
// sets the flag); 1: recompute pass (rows given by rows_map, writes lse,
// logprob, argmax and recomputed = 1; margin keeps the main-pass value);
// 2: both in one launch (the one-pass layout): the main partials of row r are
// rows r of part and its exact partials rows B + r; the flag decided by the
// main margin picks which merge gives lse, logprob and argmax.
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
  LmRow m = lm_merge_row(part + (size_t)r * n_chunks, n_chunks, lane);
  const int orow = rows_map ? rows_map[r] : r;
  const int tg = target ? target[orow] : -1;
  if (mode_recompute == 1) {
    if (lane != 0) return;
    lse[orow] = m.L;
    logprob[orow] = (tg >= 0 && m.has) ? m.zt - m.L : m.v1 - m.L;
    argmax[orow] = m.i1;
    recomputed[orow] = 1;
    return;
  }
  const float mg = m.v1 - m.v2;
  const bool f = thresh > 0.f && mg < thresh;  // uniform across the warp
  if (mode_recompute == 2 && f) m = lm_merge_row(part + (size_t)(B + r) * n_chunks, n_chunks, lane);
  if (lane != 0) return;
  lse[orow] = m.L;
  logprob[orow] = (tg >= 0 && m.has) ? m.zt - m.L : m.v1 - m.L;
  argmax[orow] = m.i1;
  margin[orow] = mg;
  if (flag) flag[orow] = f;
  recomputed[orow] = mode_recompute == 2 && f;
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
