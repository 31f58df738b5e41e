/*
 * Seeded synthetic inputs for the DSA hot path (indexer -> top-k -> sparse attention).
 *
 * This file holds no arithmetic of the method itself: it only draws numbers.  Both the
 * CPU oracle checks and the CUDA path take their inputs from here (through the Python
 * wrapper in synth/__init__.py), so the two sides always see the same bf16 values.
 *
 * Random numbers
 *   Counter-based: element i of a stream keyed by (seed, stream_key) uses the outputs
 *   2i and 2i+1 of a SplitMix64 sequence (Steele, Lea, Flood, "Fast splittable
 *   pseudorandom number generators", OOPSLA 2014) started at a per-stream state, turned
 *   into two uniforms in (0,1] with 53 bits each, then into one N(0,1) sample with the
 *   Box-Muller transform (cosine branch).  The sample is rounded to float, then to bf16
 *   with round-to-nearest-even.  Any element can be regenerated on its own, in parallel.
 *
 * Token layouts (the structure of the pages' long-video inputs)
 *   Each token t is either "text" (iid N(0,1)) or belongs to a frame block B.  For a
 *   block-structured tensor, a frame token's value in channel c is
 *       mean[B, c] + 0.5 * noise[t, c]
 *   with mean and noise both N(0,1) draws from two different streams; computed in
 *   float, then rounded to bf16.  Tensors that are not block-structured are iid for
 *   every token.
 *     SYNTH_LAYOUT_IID            every token is text
 *     SYNTH_LAYOUT_BLOCKS  (p0)   block = t / p0                     (equal frames)
 *     SYNTH_LAYOUT_FRAME_TEXT (p0,p1)  period p0+p1: p0 frame tokens then p1 text tokens
 *     SYNTH_LAYOUT_TEXT_FRAME (p0,p1)  period p0+p1: p0 text tokens then p1 frame tokens
 *   A token at or beyond `iid_from` is text whatever the layout says (decode tails).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SYNTH_LAYOUT_IID 0
#define SYNTH_LAYOUT_BLOCKS 1
#define SYNTH_LAYOUT_FRAME_TEXT 2
#define SYNTH_LAYOUT_TEXT_FRAME 3

static const uint64_t kGamma = 0x9E3779B97F4A7C15ULL;

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Start state of a stream: two SplitMix64 outputs mixed from the seed and the key. */
static inline uint64_t stream_state(uint64_t seed, uint64_t stream_key) {
    return mix64(mix64(seed + kGamma) ^ (stream_key * kGamma + 0x632BE59BD9B4E019ULL));
}

/* n-th output (n >= 0) of the SplitMix64 sequence whose state starts at `state`. */
static inline uint64_t splitmix_at(uint64_t state, uint64_t n) {
    return mix64(state + (n + 1) * kGamma);
}

static inline double normal_at(uint64_t state, uint64_t i) {
    uint64_t a = splitmix_at(state, 2 * i);
    uint64_t b = splitmix_at(state, 2 * i + 1);
    double u1 = ((double)(a >> 11) + 1.0) * (1.0 / 9007199254740992.0); /* (0,1] */
    double u2 = ((double)(b >> 11) + 1.0) * (1.0 / 9007199254740992.0);
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}

/* float -> bf16 bits, round to nearest even (NaN is never produced here). */
static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* Block id of token t, or -1 for a text token. */
static inline int64_t block_of(int64_t t, int layout, int64_t p0, int64_t p1, int64_t iid_from) {
    if (iid_from >= 0 && t >= iid_from) return -1;
    switch (layout) {
    case SYNTH_LAYOUT_BLOCKS:
        return t / p0;
    case SYNTH_LAYOUT_FRAME_TEXT: {
        int64_t per = p0 + p1, pos = t % per;
        return pos < p0 ? t / per : -1;
    }
    case SYNTH_LAYOUT_TEXT_FRAME: {
        int64_t per = p0 + p1, pos = t % per;
        return pos >= p0 ? t / per : -1;
    }
    default:
        return -1;
    }
}

/*
 * Fill out[(t - t0) * C + c] for t in [t0, t0 + n_tok), c in [0, C) with bf16 bits.
 * noise_key / mean_key: stream keys of the per-token noise and of the per-block means.
 * structured == 0 makes every token iid N(0,1) whatever the layout.
 */
void synth_fill_bf16(uint16_t *out, int64_t t0, int64_t n_tok, int64_t C, uint64_t seed,
                     uint64_t noise_key, uint64_t mean_key, int structured, int layout,
                     int64_t p0, int64_t p1, int64_t iid_from) {
    uint64_t ns = stream_state(seed, noise_key);
    uint64_t ms = stream_state(seed, mean_key);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n_tok; ++i) {
        int64_t t = t0 + i;
        int64_t blk = structured ? block_of(t, layout, p0, p1, iid_from) : -1;
        for (int64_t c = 0; c < C; ++c) {
            double z = normal_at(ns, (uint64_t)(t * C + c));
            float v;
            if (blk < 0) {
                v = (float)z;
            } else {
                float mean = (float)normal_at(ms, (uint64_t)(blk * C + c));
                v = mean + 0.5f * (float)z;
            }
            out[i * C + c] = f32_to_bf16_rne(v);
        }
    }
}

/* Block id per token (for tests and statistics). */
void synth_block_ids(int64_t *out, int64_t t0, int64_t n_tok, int layout, int64_t p0, int64_t p1,
                     int64_t iid_from) {
    for (int64_t i = 0; i < n_tok; ++i) out[i] = block_of(t0 + i, layout, p0, p1, iid_from);
}

/* Uniform integers in [0, hi) (sampling of query rows for sampled checks). */
void synth_uniform_int(int64_t *out, int64_t n, int64_t hi, uint64_t seed, uint64_t key) {
    uint64_t s = stream_state(seed, key);
    for (int64_t i = 0; i < n; ++i) out[i] = (int64_t)(splitmix_at(s, (uint64_t)i) % (uint64_t)hi);
}
