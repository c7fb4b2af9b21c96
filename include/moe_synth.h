/*
 * moe_synth.h -- device-side seeded input generator (test and benchmark utility).
 *
 * Not part of the layer: it fills device buffers with the same counter-based
 * streams that the host generator (Python package `synth`) produces, so that
 * full-size inputs can be made on the GPU while the host regenerates any slice of
 * them bit for bit.  Element i of a stream with seed s:
 *   word(j)     = SplitMix64 finaliser of (s + (j + 1) * 0x9E3779B97F4A7C15) mod 2^64
 *                 (Steele, Lea & Flood, OOPSLA 2014);
 *   normal      = (sum of the twelve 16-bit fields of words 3i, 3i+1, 3i+2 - 393210) / 65536
 *                 (Irwin-Hall sum of twelve uniforms minus six), times `stddev` in float64,
 *                 rounded to fp32 then to bf16 (nearest even);
 *   uniform     = lo + (hi - lo) * (word(i) >> 11) * 2^-53 in float64 (no fused
 *                 multiply-add), rounded to fp32 then to bf16.
 * Elements start .. start+n-1 are written to out[0 .. n-1] (device, bf16 bits).
 * Errors: MOE_ERR_INVALID_ARG for a null pointer or n < 0, start < 0.
 */
#ifndef MOE_SYNTH_H_
#define MOE_SYNTH_H_

#include "moe.h"

#ifdef __cplusplus
extern "C" {
#endif

moe_status_t moe_synth_normal_bf16(uint16_t* out, int64_t n, int64_t start, uint64_t seed,
                                   double stddev, moe_stream_t stream);

moe_status_t moe_synth_uniform_bf16(uint16_t* out, int64_t n, int64_t start, uint64_t seed,
                                    double lo, double hi, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_SYNTH_H_ */
