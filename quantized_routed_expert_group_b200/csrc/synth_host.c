/*
 * synth_host.c -- host side of the seeded synthetic-input generator.
 *
 * Holds no arithmetic of the MoE method: it only turns (seed, tensor id,
 * element index) into fp32 numbers.  The CUDA library carries its own copy of
 * the same counter-based generator (synth.cu) so that multi-GB expert weights
 * can be drawn in device memory; tests check that both give identical bits.
 *
 * Generator: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014), used counter-style: the n-th output of a
 * SplitMix64 stream seeded with s is mix(s + (n+1)*GAMMA).
 *   key(seed, tid)    = n=tid output of the stream seeded with `seed`
 *   word(seed,tid,n)  = n-th output of the stream seeded with key(seed, tid)
 * normal-like(i): the twelve 16-bit fields of words 3i, 3i+1, 3i+2 are summed
 *   (Irwin-Hall sum of 12 uniforms, mean 0 and variance 1 after centring):
 *   z = (S - 393210) / 65536 (exact in fp32), value = z * sigma (one fp32
 *   multiply, round to nearest).
 * uniform(i): f = (word(i) >> 40) * 2^-24 (exact), value = f * width + lo
 *   (fp32 multiply then fp32 add).
 * Built with -ffp-contract=off so the multiply and add stay separate.
 */
#include <stdint.h>

#define SM_GAMMA 0x9E3779B97F4A7C15ULL

static uint64_t sm_mix(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t synth_key(uint64_t seed, uint64_t tid) { return sm_mix(seed + (tid + 1) * SM_GAMMA); }

uint64_t synth_word(uint64_t key, uint64_t n) { return sm_mix(key + (n + 1) * SM_GAMMA); }

void synth_words(uint64_t seed, uint64_t tid, uint64_t n0, int64_t n, uint64_t *out)
{
    uint64_t key = synth_key(seed, tid);
    for (int64_t i = 0; i < n; ++i) out[i] = synth_word(key, n0 + (uint64_t)i);
}

void synth_normal(uint64_t seed, uint64_t tid, int64_t offset, int64_t n, float sigma, float *out)
{
    uint64_t key = synth_key(seed, tid);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        uint64_t e = (uint64_t)(offset + i);
        int64_t s = 0;
        for (int w = 0; w < 3; ++w) {
            uint64_t r = synth_word(key, 3 * e + (uint64_t)w);
            s += (int64_t)(r & 0xFFFF) + (int64_t)((r >> 16) & 0xFFFF) +
                 (int64_t)((r >> 32) & 0xFFFF) + (int64_t)(r >> 48);
        }
        float z = (float)(s - 393210) / 65536.0f;
        out[i] = z * sigma;
    }
}

void synth_uniform(uint64_t seed, uint64_t tid, int64_t offset, int64_t n, float lo, float width, float *out)
{
    uint64_t key = synth_key(seed, tid);
    for (int64_t i = 0; i < n; ++i) {
        uint64_t r = synth_word(key, (uint64_t)(offset + i));
        float f = (float)(r >> 40) * 0x1p-24f;
        float v = f * width;
        out[i] = v + lo;
    }
}
