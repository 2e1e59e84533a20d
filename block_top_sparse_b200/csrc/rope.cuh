// rope.cuh -- rotary position embedding of the queries and keys, in place.
//
// The paper's models carry rotary positions on q and k (section 6), and the
// continued training at 32k uses a RoPE scaling factor of 4, which stretches
// the rotation periods (Appendix K).  Rotate-half form: for i < d/2 the pair
// (x_i, x_{i+d/2}) turns by a(t, i) = (pos0 + t) * base^(-2i/d) / factor;
// `transpose` turns by -a, which carries gradients back through the rotation
// (the rotation is orthogonal).  The pooled keys, the selection and both
// attention streams then read the rotated q and k.
//
// One CTA per (sequence, 32 positions): the angles' cosines and sines are
// computed once in fp64 (positions reach 2^23 and more, far beyond what an
// fp32 angle resolves) and shared by every head; each thread then rotates 8
// pairs of a row with 16-byte loads and stores.  Bandwidth-bound: one read and
// one write of the tensor.
#pragma once

#include "pool_select.cuh"

namespace ssa {

constexpr int kRopeRows = 32;  // positions per CTA

template <typename T>
__global__ void __launch_bounds__(256) rope_kernel(T *__restrict__ X, int heads, int T_len, int d, int pos0,
                                                   double log2_base, double inv_factor, int transpose) {
    __shared__ float cs[kRopeRows][64], sn[kRopeRows][64];  // d / 2 <= 64
    const int half = d / 2;
    const int b = blockIdx.y, t0 = blockIdx.x * kRopeRows;
    for (int e = threadIdx.x; e < kRopeRows * half; e += blockDim.x) {
        const int tt = e / half, i = e % half;
        const double a = static_cast<double>(pos0 + t0 + tt) * exp2(-2.0 * i / d * log2_base) * inv_factor;
        double sv, cv;
        sincos(transpose ? -a : a, &sv, &cv);
        cs[tt][i] = static_cast<float>(cv);
        sn[tt][i] = static_cast<float>(sv);
    }
    __syncthreads();
    constexpr int V = 16 / sizeof(T);  // elements per 16-byte access
    const int units = half / V;        // 16-byte units per half row
    const int rows_per_pass = blockDim.x / units;
    const int u = threadIdx.x % units, rr = threadIdx.x / units;
    const int nt = min(kRopeRows, T_len - t0);
    for (int row = rr; row < heads * kRopeRows; row += rows_per_pass) {
        const int h = row / kRopeRows, tt = row % kRopeRows;
        if (tt >= nt) continue;
        T *x = X + ((static_cast<size_t>(b) * heads + h) * T_len + t0 + tt) * d + u * V;
        float a[V], c[V];
        if constexpr (sizeof(T) == 2) {
            const uint4 w0 = *reinterpret_cast<const uint4 *>(x), w1 = *reinterpret_cast<const uint4 *>(x + half);
            const uint32_t p0[4] = {w0.x, w0.y, w0.z, w0.w}, p1[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                a[2 * q] = __uint_as_float(p0[q] << 16);
                a[2 * q + 1] = __uint_as_float(p0[q] & 0xFFFF0000u);
                c[2 * q] = __uint_as_float(p1[q] << 16);
                c[2 * q + 1] = __uint_as_float(p1[q] & 0xFFFF0000u);
            }
        } else {
            const float4 w0 = *reinterpret_cast<const float4 *>(x), w1 = *reinterpret_cast<const float4 *>(x + half);
            a[0] = w0.x, a[1] = w0.y, a[2] = w0.z, a[3] = w0.w;
            c[0] = w1.x, c[1] = w1.y, c[2] = w1.z, c[3] = w1.w;
        }
        float y0[V], y1[V];
#pragma unroll
        for (int v = 0; v < V; ++v) {
            const float co = cs[tt][u * V + v], si = sn[tt][u * V + v];
            y0[v] = a[v] * co - c[v] * si;
            y1[v] = a[v] * si + c[v] * co;
        }
        if constexpr (sizeof(T) == 2) {
            *reinterpret_cast<uint4 *>(x) = make_uint4(pack_bf16x2(y0[0], y0[1]), pack_bf16x2(y0[2], y0[3]),
                                                       pack_bf16x2(y0[4], y0[5]), pack_bf16x2(y0[6], y0[7]));
            *reinterpret_cast<uint4 *>(x + half) = make_uint4(pack_bf16x2(y1[0], y1[1]), pack_bf16x2(y1[2], y1[3]),
                                                              pack_bf16x2(y1[4], y1[5]), pack_bf16x2(y1[6], y1[7]));
        } else {
            *reinterpret_cast<float4 *>(x) = make_float4(y0[0], y0[1], y0[2], y0[3]);
            *reinterpret_cast<float4 *>(x + half) = make_float4(y1[0], y1[1], y1[2], y1[3]);
        }
    }
}

}  // namespace ssa
