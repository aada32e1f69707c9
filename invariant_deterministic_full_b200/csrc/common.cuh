// Shared helpers of libbi: status/error state, tensor-map encoding, and the
// inline-PTX primitives the kernels use (mbarrier, TMA, ldmatrix, mma.sync).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <string>
#include <utility>

#include "../../include/bi.h"

namespace bi {

// ------------------------------------------------------------------ errors
int set_error(int status, const char* fmt, ...);
void clear_error();

#define BI_CHECK_CUDA(call)                                                                   \
  do {                                                                                        \
    cudaError_t e_ = (call);                                                                  \
    if (e_ != cudaSuccess) return ::bi::set_error(BI_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)
extern long long g_launches;  // host-side count of kernels launched by the library
#define BI_CHECK_LAUNCH()            \
  do {                               \
    ++::bi::g_launches;              \
    BI_CHECK_CUDA(cudaGetLastError()); \
  } while (0)
#define BI_REQUIRE(cond, status, ...)                 \
  do {                                                \
    if (!(cond)) return ::bi::set_error(status, __VA_ARGS__); \
  } while (0)
#define BI_TRY(expr)             \
  do {                           \
    int s_ = (expr);             \
    if (s_ != BI_OK) return s_;  \
  } while (0)

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
int num_sms();  // of the current device (cached per device)
bool pdl_enabled();  // programmatic dependent launch (env BI_PDL=0 turns it off)
// Every kernel runs with the largest shared-memory carveout, so all kernels
// share one L1 / shared-memory split: an SM still holding CTAs of a kernel
// with little shared memory (the norm) then also takes CTAs of the GEMM or
// attention kernel launched behind it instead of waiting to drain.  Sets the
// attribute the first time a thread launches `kern` on the current device.
int ensure_carveout(const void* kern);

// Launch a library kernel on `st`, with programmatic stream serialisation
// allowed (see pdl_wait / pdl_trigger), counting it in g_launches.
template <typename... KArgs, typename... Args>
int launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  BI_TRY(ensure_carveout(reinterpret_cast<const void*>(kern)));
  BI_CHECK_CUDA(cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...));
  BI_CHECK_LAUNCH();
  return BI_OK;
}

// Device-side error word: kernels set bits here instead of trapping when a
// bounded wait runs out or an index fails its check.
enum : unsigned { DEVERR_TIMEOUT = 1u, DEVERR_CAPACITY = 2u, DEVERR_INDEX = 4u };
__device__ unsigned g_dev_error = 0;  // one translation unit: defined here
__device__ unsigned g_dev_site = 0;   // site code of the first wait that ran out (0: none)
__device__ __forceinline__ void dev_flag(unsigned bit) { atomicOr(&g_dev_error, bit); }

// Tensor maps (TMA descriptors), encoded through the driver entry point.
int encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, int elem_bytes, const void* base, uint64_t inner,
                   uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                   CUtensorMapSwizzle swizzle);
// 3-D view: dims[0] contiguous elements; strides in bytes of dims 1 and 2.
int encode_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, const uint64_t dims[3],
                   const uint64_t strides[2], const uint32_t box[3], CUtensorMapSwizzle swizzle);

// ------------------------------------------------------------------ PTX helpers
// Programmatic dependent launch.  Every kernel of the library calls pdl_wait()
// before it reads anything an earlier kernel wrote and before it writes
// anything (so the chain of completions stays transitive), then pdl_trigger()
// so the next kernel may be scheduled and run its independent prologue
// (barrier set-up, weight prefetch) while this one finishes: at once, except
// in the norm, which first lets its own few loads land.  Both are no-ops for a
// kernel launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: returns false (and flags the device error word) if the phase
// does not complete within the iteration limit (each try_wait suspends for a
// hardware-chosen interval, so the limit is seconds, never forever).
// Bounded waits: a wait gives up after kWaitNs of wall-clock time (the
// global nanosecond timer), whatever each try_wait costs.
constexpr uint64_t kWaitNs = 1000000000ull;  // 1 s
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// site: which wait ran out, reported in bits 8..15 of bi_device_error's flags.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned site = 0) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitNs) break;
  }
  dev_flag(DEVERR_TIMEOUT);
  atomicCAS(&g_dev_site, 0u, site);
  return false;
}
enum : unsigned {
  SITE_GEMM_EMPTY = 0x11, SITE_GEMM_FULL = 0x12, SITE_GEMM_DRAIN = 0x13,
  SITE_ATTN_CORE = 0x21, SITE_ATTN_TC = 0x22, SITE_SELFTEST = 0x31
};

// 3D tiled TMA load (coordinates innermost first).
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}
// The same copy with an L2 eviction policy (see l2_evict_first).
__device__ __forceinline__ void tma_load_3d_hint(void* smem_dst, const CUtensorMap* map, int c0, int c1, int c2,
                                                 uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, "
      "%3, %4}], [%5], %6;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
// L2 policy for data read once per decode step (weights, KV rows): its lines
// are the first to be evicted, so they do not push out the small activations
// and residual rows that the next kernels read back.
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
// D = A(16x16 bf16, row) * B(16x8 bf16, col) + D, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Address of the 16-byte chunk `chunk` of row `row` inside a TMA tile written
// with CU_TENSOR_MAP_SWIZZLE_128B (128-byte rows, tile base 1024-byte aligned):
// chunk c of row r lives at chunk position c ^ (r & 7).
__device__ __forceinline__ uint32_t swz128(uint32_t tile_base, int row, int chunk) {
  return tile_base + row * 128 + ((chunk ^ (row & 7)) << 4);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Store one activation value in the mode's dtype (bf16: round to nearest even).
__device__ __forceinline__ void store_act(void* base, size_t idx, float v, bool f32) {
  if (f32)
    reinterpret_cast<float*>(base)[idx] = v;
  else
    reinterpret_cast<uint16_t*>(base)[idx] = f32_to_bf16_bits(v);
}
__device__ __forceinline__ float load_act(const void* base, size_t idx, bool f32) {
  return f32 ? reinterpret_cast<const float*>(base)[idx]
             : bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(base)[idx]);
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }

// Rotate-half RoPE of the pair (a, b) = (x[i], x[i + d/2]) by (c, s):
// a' = a c - b s, b' = b c + a s, with the rounding spelled out (the second
// product rounded, the first fused) so that every kernel that rotates -- the
// two GEMM epilogues and the standalone kernel -- gives the same bits; left to
// the compiler, a*c - b*s may be contracted differently in each.
__device__ __forceinline__ void rope_rotate(float a, float b, float c, float s, float& ra, float& rb) {
  ra = __fmaf_rn(a, c, -__fmul_rn(b, s));
  rb = __fmaf_rn(b, c, __fmul_rn(a, s));
}

// Fixed butterfly sum over the 32 lanes: every lane ends with the same value
// (each level adds the same two operands, only their order differs, and fp
// addition is commutative).
__device__ __forceinline__ float warp_sum_fixed(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace bi
