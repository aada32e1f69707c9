/* Seeded synthetic input generator (host side).
 *
 * Shared by the oracle and the GPU harness as DATA only: it holds none of the
 * decoder's arithmetic.  Definitions (the device-side twin in the package's
 * csrc/synth_fill.cu implements the same published definitions independently):
 *
 *   SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
 *   generators", OOPSLA 2014; constants as published by Vigna):
 *     mix(z)  : z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
 *               z = (z ^ (z >> 27)) * 0x94D049BB133111EB
 *               return z ^ (z >> 31)
 *     draw(key, i) = mix(key + (i + 1) * 0x9E3779B97F4A7C15)   (counter-based)
 *   stream key(seed, stream) = mix(seed ^ mix(stream + 0x632BE59BD9B4E019))
 *
 *   normal(key, i): Irwin-Hall sum of twelve 16-bit uniforms (the four 16-bit
 *     fields of draw(key,3i), draw(key,3i+1), draw(key,3i+2)), centred and
 *     scaled to unit variance:  z = (S - 393210) / sqrt(65536^2 - 1).
 *     Integer sum + one IEEE division: bit-identical on any IEEE machine.
 *   weight value : bf16_rne( float_rne( z * std ) )
 *   token id     : draw(key, i) mod V
 */
#include <stdint.h>
#include <string.h>

#define SM_GAMMA 0x9E3779B97F4A7C15ULL
#define IH_SD 65535.99999237060546875 /* sqrt(65536^2 - 1) rounded to double */

static inline uint64_t sm_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}
uint64_t synth_key(uint64_t seed, uint64_t stream) {
  return sm_mix(seed ^ sm_mix(stream + 0x632BE59BD9B4E019ULL));
}
static inline uint64_t sm_draw(uint64_t key, uint64_t i) { return sm_mix(key + (i + 1) * SM_GAMMA); }

uint64_t synth_draw(uint64_t key, uint64_t i) { return sm_draw(key, i); }

static inline double ih_normal(uint64_t key, uint64_t i) {
  int64_t s = 0;
  for (int j = 0; j < 3; ++j) {
    uint64_t d = sm_draw(key, 3 * i + (uint64_t)j);
    s += (int64_t)(d & 0xFFFF) + (int64_t)((d >> 16) & 0xFFFF) + (int64_t)((d >> 32) & 0xFFFF) + (int64_t)(d >> 48);
  }
  return (double)(s - 393210) / IH_SD;
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u; memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)((u >> 16) | ((u & 0xFFFF) ? 0x40 : 0));
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* n standard normals (doubles) of stream key, elements [start, start+n). */
void synth_normal_f64(uint64_t key, uint64_t start, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = ih_normal(key, start + (uint64_t)i);
}
/* bf16 bit patterns of std * normal, elements [start, start+n). */
void synth_normal_bf16(uint64_t key, uint64_t start, int64_t n, double std, uint16_t* out) {
#pragma omp parallel for schedule(static) if (n > 65536)
  for (int64_t i = 0; i < n; ++i) {
    double z = ih_normal(key, start + (uint64_t)i);
    out[i] = f32_to_bf16_rne((float)(z * std));
  }
}
/* token ids uniform in [0, V). */
void synth_tokens(uint64_t key, uint64_t start, int64_t n, int64_t vocab, int32_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = (int32_t)(sm_draw(key, start + (uint64_t)i) % (uint64_t)vocab);
}
