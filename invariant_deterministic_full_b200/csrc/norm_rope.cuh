// RMSNorm (fused residual add), RoPE + KV-cache append, embedding gather.
#pragma once
#include "common.cuh"

namespace bi {

constexpr int NORM_THREADS = 128;
constexpr int NORM_MAX_CHUNKS = 16;  // 8-element chunks per thread: H <= 128*16*8 = 16384

// Load/store 8 consecutive activation values (bf16: one 16-byte access; f32: two).
__device__ __forceinline__ void load8(const void* base, size_t off, bool f32, float* v) {
  if (f32) {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + off);
    const float4 a = p[0], b = p[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 u = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(base) + off);
    v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
    v[4] = bf16lo(u.z); v[5] = bf16hi(u.z); v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
  }
}
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  return (uint32_t)f32_to_bf16_bits(a) | ((uint32_t)f32_to_bf16_bits(b) << 16);
}
__device__ __forceinline__ void store8(void* base, size_t off, bool f32, const float* v) {
  if (f32) {
    float4* p = reinterpret_cast<float4*>(reinterpret_cast<float*>(base) + off);
    p[0] = make_float4(v[0], v[1], v[2], v[3]);
    p[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
    *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(base) + off) =
        make_uint4(pack2(v[0], v[1]), pack2(v[2], v[3]), pack2(v[4], v[5]), pack2(v[6], v[7]));
  }
}
// Value as stored in the activation dtype (bf16: round to nearest even).
__device__ __forceinline__ float as_stored(float v, bool f32) {
  return f32 ? v : bf16_bits_to_f32(f32_to_bf16_bits(v));
}

// One row, NORM_THREADS threads (tid = 0 .. NORM_THREADS-1).  Thread i owns
// the 8-element chunks i, i + NORM_THREADS, ... of the row (at most CPT of
// them, held in registers: every load of the thread is issued at once); its
// partial sum of squares runs over them in ascending order, then a fixed
// xor-butterfly inside each warp, then the warp sums are added in ascending
// warp order (every thread repeats that same sequential sum).  r = x
// (+ res_in, rounded as stored), written to res_out; y = (r * inv) * gamma.
// `bar` synchronises the NORM_THREADS threads (a CTA barrier, or a named
// barrier inside a larger CTA).  The row waits for the previous kernel
// (pdl_wait) before it reads x; with `early` the residual row and gamma, which
// the caller guarantees were written before the previous kernel, are loaded
// before that wait.
template <int CPT, typename Bar>
__device__ __forceinline__ void rmsnorm_row(const void* __restrict__ x, const void* __restrict__ res_in,
                                            void* __restrict__ res_out, const uint16_t* __restrict__ gamma,
                                            void* __restrict__ y, float* __restrict__ y32, int row, int H, float eps,
                                            int f32, int tid, float* wsum, Bar bar, bool early) {
  const int nch = H / 8;
  const size_t rbase = (size_t)row * H;
  float v[CPT][8], r[CPT][8];
  uint4 gu[CPT];
  auto load_res_gamma = [&]() {
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
      const int ch = tid + i * NORM_THREADS;
      if (ch < nch) {
        if (res_in) load8(res_in, rbase + ch * 8, f32, r[i]);
        gu[i] = *reinterpret_cast<const uint4*>(gamma + ch * 8);
      }
    }
  };
  if (early) load_res_gamma();
  pdl_wait();
  if (!early) load_res_gamma();
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const int ch = tid + i * NORM_THREADS;
    if (ch < nch) {
      load8(x, rbase + ch * 8, f32, v[i]);
      if (res_in) {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[i][j] = as_stored(v[i][j] + r[i][j], f32);
      }
    }
  }
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < CPT; ++i)
    if (tid + i * NORM_THREADS < nch) {
#pragma unroll
      for (int j = 0; j < 8; ++j) ss = fmaf(v[i][j], v[i][j], ss);
    }
  ss = warp_sum_fixed(ss);
  if ((tid & 31) == 0) wsum[tid >> 5] = ss;
  bar();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < NORM_THREADS / 32; ++w) tot += wsum[w];
  const float inv = 1.0f / sqrtf(tot / (float)H + eps);
  bar();  // wsum may be reused by the next row
  // Every load of the row has landed: the next kernel may now be scheduled
  // (its weight prefetch would otherwise queue ahead of these loads).
  pdl_trigger();
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const int ch = tid + i * NORM_THREADS;
    if (ch < nch) {
      if (res_out) store8(res_out, rbase + ch * 8, f32, v[i]);
      const float gm[8] = {bf16lo(gu[i].x), bf16hi(gu[i].x), bf16lo(gu[i].y), bf16hi(gu[i].y),
                           bf16lo(gu[i].z), bf16hi(gu[i].z), bf16lo(gu[i].w), bf16hi(gu[i].w)};
      float o[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) o[j] = v[i][j] * inv * gm[j];
      store8(y, rbase + ch * 8, f32, o);
      if (y32) {
        float4* p = reinterpret_cast<float4*>(y32 + rbase + ch * 8);
        p[0] = make_float4(o[0], o[1], o[2], o[3]);
        p[1] = make_float4(o[4], o[5], o[6], o[7]);
      }
    }
  }
}

// One CTA per row (see rmsnorm_row, which waits for the previous kernel and
// releases the next once the row's loads have landed); CPT: chunks per
// thread, the smallest of 1, 2, 4, 8, 16 that covers the row.  early: see
// rmsnorm_row (the decode step, where the residual row was written by a norm
// at least two kernels back).
template <int CPT>
__global__ void __launch_bounds__(NORM_THREADS)
    rmsnorm_kernel(const void* __restrict__ x, const void* __restrict__ res_in, void* __restrict__ res_out,
                   const uint16_t* __restrict__ gamma, void* __restrict__ y, float* __restrict__ y32, int H, float eps,
                   int f32, int early) {
  if (!early) {
    // Before the dependency wait, request the row's residual and gamma into
    // L2 (a prefetch returns no value, so it cannot observe data that an
    // earlier kernel is still writing): after the wait the row's loads find
    // them there instead of queuing for DRAM.
    const int esz = f32 ? 4 : 2;
    const int rlines = res_in ? H * esz / 128 : 0, glines = H * 2 / 128;
    for (int i = threadIdx.x; i < rlines + glines; i += NORM_THREADS) {
      const char* pa = i < rlines ? reinterpret_cast<const char*>(res_in) + (size_t)blockIdx.x * H * esz + i * 128
                                  : reinterpret_cast<const char*>(gamma) + (size_t)(i - rlines) * 128;
      asm volatile("prefetch.global.L2 [%0];" ::"l"(pa));
    }
  }
  __shared__ float wsum[NORM_THREADS / 32];
  rmsnorm_row<CPT>(x, res_in, res_out, gamma, y, y32, blockIdx.x, H, eps, f32, threadIdx.x, wsum,
                   [] { __syncthreads(); }, early != 0);
}
__host__ __device__ constexpr int norm_cpt(int H) {
  return H / 8 <= NORM_THREADS ? 1 : H / 8 <= 2 * NORM_THREADS ? 2 : H / 8 <= 4 * NORM_THREADS ? 4
         : H / 8 <= 8 * NORM_THREADS ? 8 : 16;
}

// Row of element i of a head (size d) in the "paired" QKV layout: within every
// 32-row block b, rows 0..15 hold elements 16b.. and rows 16..31 their
// rotate-half partners d/2 + 16b ...
__host__ __device__ inline int paired_row(int i, int d) {
  const int half = d >> 1;
  return i < half ? 32 * (i >> 4) + (i & 15) : 32 * ((i - half) >> 4) + 16 + ((i - half) & 15);
}

// Rotate-half RoPE of q and k heads, then q -> q_out and k, v -> cache row
// (slot, layer, head, pos).  One CTA per token.  table: [max_pos][d/2][2].
// paired != 0: the q and k heads of qkv are in the paired row order.
__global__ void rope_append_kernel(const float* __restrict__ qkv, const float* __restrict__ table, int table_max_pos,
                                   void* __restrict__ q_out, void* __restrict__ kc, void* __restrict__ vc,
                                   const int32_t* __restrict__ slot, const int32_t* __restrict__ pos, int Hq, int Hkv,
                                   int d, int layer, int n_layers, int n_slots, int cap, int f32, int paired) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  const int half = d / 2;
  const int p = pos[t], s = slot[t];
  const bool ok = p >= 0 && p < cap && p < table_max_pos && s >= 0 && s < n_slots;
  if (!ok) {
    if (threadIdx.x == 0) dev_flag(DEVERR_CAPACITY);
    return;
  }
  const int QD = Hq * d, KD = Hkv * d;
  const float* row = qkv + (size_t)t * (QD + 2 * KD);
  const float* cs = table + (size_t)p * d;  // [half][2]
  // q and k rotations: pairs (i, i + half) of each head
  const int npairs = (Hq + Hkv) * half;
  for (int idx = threadIdx.x; idx < npairs; idx += blockDim.x) {
    const int h = idx / half, i = idx % half;
    const float c = cs[2 * i], sn = cs[2 * i + 1];
    const int ia = paired ? paired_row(i, d) : i, ib = paired ? paired_row(i + half, d) : i + half;
    const float a = row[h * d + ia], b = row[h * d + ib];
    float ra, rb;
    rope_rotate(a, b, c, sn, ra, rb);
    if (h < Hq) {
      store_act(q_out, (size_t)t * QD + h * d + i, ra, f32);
      store_act(q_out, (size_t)t * QD + h * d + i + half, rb, f32);
    } else {
      const int hk = h - Hq;
      const size_t crow = (((size_t)s * n_layers + layer) * Hkv + hk) * cap + p;
      store_act(kc, crow * d + i, ra, f32);
      store_act(kc, crow * d + i + half, rb, f32);
    }
  }
  for (int idx = threadIdx.x; idx < KD; idx += blockDim.x) {
    const int hk = idx / d, e = idx % d;
    const size_t crow = (((size_t)s * n_layers + layer) * Hkv + hk) * cap + p;
    store_act(vc, crow * d + e, row[QD + KD + idx], f32);
  }
}

// x[t][:] = E[ids[t]][:] in the activation dtype.
// E: bf16 (ET = uint16_t) or f32 (ET = float, FP32-storage mode) [V][H].
template <typename ET>
__global__ void embed_kernel(const int32_t* __restrict__ ids, const ET* __restrict__ E, void* __restrict__ x,
                             int H, int V, int f32) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  const int id = ids[t];
  if (id < 0 || id >= V) {
    if (threadIdx.x == 0) dev_flag(DEVERR_INDEX);
    for (int i = threadIdx.x; i < H; i += blockDim.x) store_act(x, (size_t)t * H + i, 0.f, f32);
    return;
  }
  for (int i = threadIdx.x; i < H; i += blockDim.x) {
    float v;
    if constexpr (sizeof(ET) == 2)
      v = bf16_bits_to_f32(E[(size_t)id * H + i]);
    else
      v = E[(size_t)id * H + i];
    store_act(x, (size_t)t * H + i, v, f32);
  }
}

__global__ void greedy_advance_kernel(const int32_t* __restrict__ argmax, int32_t* __restrict__ ids,
                                      int32_t* __restrict__ pos, int B) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) {
    ids[b] = argmax[b];
    pos[b] += 1;
  }
}

}  // namespace bi
