/*
 * synth.c -- seeded synthetic inputs shared by the tests, the oracle checks and
 * the benchmark.  It holds none of the attention method's arithmetic: it only
 * draws i.i.d. N(0, 1) values and rounds them to bf16.
 *
 * Generator (both published methods):
 *   - SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
 *     generators", OOPSLA 2014): state += 0x9E3779B97F4A7C15, then the output
 *     mix z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27;
 *     z *= 0x94D049BB133111EB; z ^= z >> 31.  Used counter-style: draw t of a
 *     stream whose state starts at S is mix(S + (t + 1) * gamma), so any
 *     element can be produced independently of the others.
 *   - Box-Muller (Box and Muller, 1958): for uniforms u1 in (0,1], u2 in [0,1),
 *     r = sqrt(-2 ln u1), z0 = r cos(2 pi u2), z1 = r sin(2 pi u2).
 * Stream of tensor `tensor_id` under `seed`: S = mix(seed + (tensor_id + 1) * gamma).
 * Element e uses draws 2*(e/2) and 2*(e/2)+1; even e takes z0, odd e takes z1.
 * fp32 -> bf16 is round-to-nearest-even on the bit pattern.
 */
#include <math.h>
#include <stdint.h>

#define SM_GAMMA 0x9E3779B97F4A7C15ULL

static uint64_t sm_mix(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t synth_stream_start(uint64_t seed, uint64_t tensor_id)
{
    return sm_mix(seed + (tensor_id + 1) * SM_GAMMA);
}

uint64_t synth_draw(uint64_t start, uint64_t t) { return sm_mix(start + (t + 1) * SM_GAMMA); }

static uint16_t f32_to_bf16_rne(float x)
{
    union {
        float f;
        uint32_t u;
    } v;
    v.f = x;
    uint32_t u = v.u;
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* Elements [first, first + count) of the stream; either output may be null. */
void synth_normal(uint64_t seed, uint64_t tensor_id, int64_t first, int64_t count, float* out_f32,
                  uint16_t* out_bf16)
{
    const uint64_t start = synth_stream_start(seed, tensor_id);
    const double two_pi = 6.283185307179586476925286766559;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; i++) {
        int64_t e = first + i;
        uint64_t pair = (uint64_t)e >> 1;
        uint64_t a = synth_draw(start, 2 * pair), b = synth_draw(start, 2 * pair + 1);
        double u1 = ((double)(a >> 11) + 1.0) * (1.0 / 9007199254740992.0); /* (0, 1] */
        double u2 = (double)(b >> 11) * (1.0 / 9007199254740992.0);         /* [0, 1) */
        double r = sqrt(-2.0 * log(u1));
        double z = (e & 1) ? r * sin(two_pi * u2) : r * cos(two_pi * u2);
        float zf = (float)z;
        if (out_f32)
            out_f32[i] = zf;
        if (out_bf16)
            out_bf16[i] = f32_to_bf16_rne(zf);
    }
}

/* Round an fp32 array to bf16 (round-to-nearest-even). */
void synth_round_bf16(const float* in, int64_t count, uint16_t* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; i++)
        out[i] = f32_to_bf16_rne(in[i]);
}
