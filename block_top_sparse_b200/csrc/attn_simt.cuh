// attn_simt.cuh -- CUDA-core attention for the shapes the tensor-core kernels do
// not take (fp32 inputs, or head dimension 64): one warp per query row, lanes
// split the head dimension, online softmax in fp32; the backward accumulates
// dK / dV with fp32 atomics.  Same definitions as the tensor-core path
// (paper section 3; zero gradient outside S(t), section 4.2).
#pragma once

#include "device.cuh"
#include "pool_select.cuh"

namespace ssa {

template <typename T>
__device__ __forceinline__ void store_as(T *p, float v);
template <>
__device__ __forceinline__ void store_as<float>(float *p, float v) {
    *p = v;
}
template <>
__device__ __forceinline__ void store_as<__nv_bfloat16>(__nv_bfloat16 *p, float v) {
    *p = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Iterate the attended positions u of query t (ascending): full -> 0..t,
// sparse -> tokens of the selected blocks up to t.
template <typename F>
__device__ __forceinline__ void for_each_attended(const int32_t *sel, int k, int s, int t, F &&f) {
    if (!sel) {
        for (int u = 0; u <= t; ++u) f(u);
        return;
    }
    for (int i = 0; i < k; ++i) {
        const int j = __ldg(sel + i);
        if (j < 0) continue;
        const int end = min((j + 1) * s, t + 1);
        for (int u = j * s; u < end; ++u) f(u);
    }
}

template <typename T, int DPL>
__global__ void __launch_bounds__(256) simt_fwd_kernel(const T *__restrict__ Q, const T *__restrict__ K,
                                                       const T *__restrict__ V, const int32_t *__restrict__ idx,
                                                       T *__restrict__ O, T *__restrict__ O_lo,
                                                       float *__restrict__ lse, size_t rows, int Tl, int s, int k,
                                                       float scale, int G) {
    const size_t row = static_cast<size_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    constexpr int d = DPL * 32;
    const int t = static_cast<int>(row % Tl);
    const size_t head = (row / Tl / G) * Tl;  // first row of the key/value head (and its selection)
    float q[DPL], o[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
        q[i] = to_f32(Q[row * d + lane + 32 * i]);
        o[i] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    for_each_attended(idx ? idx + (head + t) * k : nullptr, k, s, t, [&](int u) {
        const T *kr = K + (head + u) * d;
        const T *vr = V + (head + u) * d;
        float part = 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) part += q[i] * to_f32(kr[lane + 32 * i]);
        const float x = warp_sum(part) * scale;
        const float mn = fmaxf(m, x);
        const float a = expf(m - mn), p = expf(x - mn);
        l = l * a + p;
#pragma unroll
        for (int i = 0; i < DPL; ++i) o[i] = o[i] * a + p * to_f32(vr[lane + 32 * i]);
        m = mn;
    });
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
        const float v = o[i] / l;
        store_as(O + row * d + lane + 32 * i, v);
        // bf16 outputs: the rounding residual o - bf16(o), rounded to bf16 (the caller passes no O_lo for fp32)
        if (O_lo) store_as(O_lo + row * d + lane + 32 * i, v - to_f32(O[row * d + lane + 32 * i]));
    }
    if (lane == 0) lse[row] = m + logf(l);
}

template <typename T, int DPL>
__global__ void __launch_bounds__(256) simt_bwd_kernel(const T *__restrict__ Q, const T *__restrict__ K,
                                                       const T *__restrict__ V, const T *__restrict__ dO,
                                                       const int32_t *__restrict__ idx, const float *__restrict__ lse,
                                                       const float *__restrict__ Dvec, float *__restrict__ dQacc,
                                                       float *__restrict__ dKacc, float *__restrict__ dVacc,
                                                       size_t rows, int Tl, int s, int k, float scale, int G) {
    const size_t row = static_cast<size_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    constexpr int d = DPL * 32;
    const int t = static_cast<int>(row % Tl);
    const size_t head = (row / Tl / G) * Tl;  // first row of the key/value head (and its selection)
    float q[DPL], g[DPL], dq[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
        q[i] = to_f32(Q[row * d + lane + 32 * i]);
        g[i] = to_f32(dO[row * d + lane + 32 * i]);
        dq[i] = 0.f;
    }
    const float L = lse[row], Dt = Dvec[row];
    for_each_attended(idx ? idx + (head + t) * k : nullptr, k, s, t, [&](int u) {
        const T *kr = K + (head + u) * d;
        const T *vr = V + (head + u) * d;
        float kx[DPL], part = 0.f, partv = 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) {
            kx[i] = to_f32(kr[lane + 32 * i]);
            part += q[i] * kx[i];
            partv += g[i] * to_f32(vr[lane + 32 * i]);
        }
        const float x = warp_sum(part) * scale;
        const float dp = warp_sum(partv);
        const float p = expf(x - L);
        const float ds = p * (dp - Dt);
#pragma unroll
        for (int i = 0; i < DPL; ++i) {
            dq[i] += scale * ds * kx[i];
            atomicAdd(dKacc + (head + u) * d + lane + 32 * i, scale * ds * q[i]);
            atomicAdd(dVacc + (head + u) * d + lane + 32 * i, p * g[i]);
        }
    });
#pragma unroll
    for (int i = 0; i < DPL; ++i) dQacc[row * d + lane + 32 * i] = dq[i];
}

}  // namespace ssa
