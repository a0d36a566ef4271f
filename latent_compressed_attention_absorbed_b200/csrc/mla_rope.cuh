// RoPE rotation shared by the generic and sm_100a kernels.
//
// Decoupled RoPE (m.lsln.cn/news/222502, section 2.3): only the small
// position part of queries and keys is rotated.  Pair (2k, 2k+1) of a d-wide
// vector turns by pos * base^(-2k/d).  The angle and its sine and cosine are
// taken in fp64 so positions up to 2^17 keep full fp32 accuracy.
#pragma once

__device__ __forceinline__ void mla_rope_pair(float x0, float x1, int k, int d, int pos, float base, float* y0,
                                              float* y1) {
    const double inv_freq = pow((double)base, -2.0 * (double)k / (double)d);
    double s, c;
    sincos((double)pos * inv_freq, &s, &c);
    *y0 = (float)((double)x0 * c - (double)x1 * s);
    *y1 = (float)((double)x0 * s + (double)x1 * c);
}
