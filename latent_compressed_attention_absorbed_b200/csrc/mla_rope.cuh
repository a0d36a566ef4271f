// RoPE rotation shared by the generic and sm_100a kernels.
//
// Decoupled RoPE (m.lsln.cn/news/222502, section 2.3): only the small
// position part of queries and keys is rotated.  Pair (2k, 2k+1) of a d-wide
// vector turns by pos * base^(-2k/d).  The inverse frequencies are computed
// once on the host in fp64 (RopeTable); the angle is formed and reduced to
// [-pi, pi] in fp64, so that positions up to 2^17 keep full fp32 accuracy,
// and its sine and cosine are taken in fp32.
#pragma once

namespace mla {

struct RopeTable {
    double inv_freq[64];  // base^(-2k/d) for k < d/2 (d <= 128)
};

}  // namespace mla

__device__ __forceinline__ void mla_rope_rotate(float x0, float x1, double inv_freq, int pos, float* y0,
                                                float* y1) {
    const double a = (double)pos * inv_freq;
    const double n = rint(a * 0.15915494309189535);     // 1 / (2 pi)
    const float r = (float)fma(-n, 6.283185307179586, a);  // a - 2 pi n, |r| <= pi
    float s, c;
    sincosf(r, &s, &c);
    *y0 = x0 * c - x1 * s;
    *y1 = x0 * s + x1 * c;
}
