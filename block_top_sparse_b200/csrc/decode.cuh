// decode.cuh -- sparse decoding with a key/value cache: one new query per
// sequence, attending over the tokens of its selected blocks.
//
// The paper's kernel keeps no key/value cache, which makes its decoding slow
// (Appendix E); its inference speed claims concern this regime (section 5,
// Appendix D).  The method is the one of the training path (section 3): the
// query's own block b(t) plus the k-1 preceding blocks with the highest mean-
// pooled-key scores, attention over their tokens up to t.  What a cache adds is
// state: the pooled key of a block is computed once, when its last token
// arrives, and kept.
//
// Per call, sequence b has its new token at position L_b = cache_len[b]; its
// key and value already sit in row L_b of the caches.
//   decode_select_kernel   one CTA per (sequence, key head): scores the complete
//                          blocks j < b(L) with the group's query (fp32 sum of
//                          its G heads' rows), keeps b(L) and the top k-1 (the
//                          warp threshold search of the training path), and
//                          writes the pooled key of block b(L) into the cache
//                          when the new token completes it;
//   decode_attend_kernel   one CTA per (sequence, key head, slot): the slot's
//                          block (up to s keys, causal in the current block)
//                          against the G query heads of the group: normalised
//                          partial output and log-sum-exp in fp32;
//   decode_combine_kernel  one warp per (sequence, query head): log-sum-exp
//                          merge of the k partials.
// Decoding is bound by reading the cache (k*s keys and values and the pooled
// keys of the preceding blocks per key head), so these are CUDA-core kernels.
#pragma once

#include "pool_select.cuh"

namespace ssa {

constexpr int kDecThreads = 256;
constexpr int kDecMaxBlocks = 1024;  // the warp search holds 32 keys per lane
constexpr int kDecMaxGroup = 16;     // query heads per key head

enum : unsigned { ERR_BAD_INPUT = 6u };

__global__ void __launch_bounds__(kDecThreads) decode_select_kernel(
    const int32_t *__restrict__ cache_len, const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ Kc,
    float *__restrict__ Kbar, int32_t *__restrict__ idx, int Hk, int G, int T, int s, int k, int nb) {
    extern __shared__ float dec_sm[];
    float *qs = dec_sm;        // [128] the group's query row
    float *sc = dec_sm + 128;  // [nb] block scores
    const int bg = blockIdx.x, b = bg / Hk;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = __ldg(cache_len + b);
    int32_t *out = idx + static_cast<size_t>(bg) * k;
    if (L < 0 || L >= T) {  // nothing valid to select: report and leave an empty row
        if (threadIdx.x == 0) record_error(ERR_BAD_INPUT, 0x601);
        for (int i = threadIdx.x; i < k; i += blockDim.x) out[i] = -1;
        return;
    }
    const int bt = L / s;  // current block; blocks j < bt are complete
    for (int c = threadIdx.x; c < 128; c += blockDim.x) {
        float v = 0.f;
        for (int hi = 0; hi < G; ++hi) v += __bfloat162float(q[(static_cast<size_t>(bg) * G + hi) * 128 + c]);
        qs[c] = v;
    }
    __syncthreads();
    // scores r_j = q . Kbar_j: warp w takes blocks w, w + 8, ...; lane l dims 4l .. 4l+3
    const float4 q4 = reinterpret_cast<const float4 *>(qs)[lane];
    float *kb = Kbar + static_cast<size_t>(bg) * nb * 128;  // this key head's pooled keys
    for (int j = warp; j < bt; j += kDecThreads / 32) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(kb + static_cast<size_t>(j) * 128) + lane);
        float part = q4.x * v.x + q4.y * v.y + q4.z * v.z + q4.w * v.w;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (lane == 0) sc[j] = part;
    }
    __syncthreads();
    if (warp == 0) select_row<kDecMaxBlocks / 32>(sc, bt, min(k - 1, bt), bt, k, out, lane);
    // the new token completes block bt: its pooled key joins the cache (read from the next step on)
    if ((L + 1) % s == 0) {
        const int c = threadIdx.x & 127, half = threadIdx.x >> 7;
        const __nv_bfloat16 *kr = Kc + (static_cast<size_t>(bg) * T + static_cast<size_t>(bt) * s) * 128 + c;
        float acc = 0.f;
        for (int r = half; r < s; r += 2) acc += __bfloat162float(kr[static_cast<size_t>(r) * 128]);
        __syncthreads();  // the scores are no longer read: reuse them for the two halves
        sc[threadIdx.x] = acc;
        __syncthreads();
        if (half == 0) kb[static_cast<size_t>(bt) * 128 + c] = (sc[c] + sc[128 + c]) / static_cast<float>(s);
    }
}

// grid = (B * Hk, k): one slot's block against the group's G query heads.
__global__ void __launch_bounds__(kDecThreads) decode_attend_kernel(
    const int32_t *__restrict__ cache_len, const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ Kc,
    const __nv_bfloat16 *__restrict__ Vc, const int32_t *__restrict__ idx, float *__restrict__ opart,
    float *__restrict__ lsepart, int Hk, int G, int T, int s, int k, float scale) {
    __shared__ float qh[kDecMaxGroup][128];
    __shared__ float S[kDecMaxGroup][128];  // scores, then weights, of the block's keys (s <= 128)
    const int bg = blockIdx.x, slot = blockIdx.y, b = bg / Hk;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = __ldg(cache_len + b);
    const int j = (L >= 0 && L < T) ? __ldg(idx + static_cast<size_t>(bg) * k + slot) : -1;
    const size_t prow0 = (static_cast<size_t>(bg) * G) * k + slot;  // partial of query head (bg*G + hi): + hi * k
    if (j < 0) {
        for (int hi = threadIdx.x; hi < G; hi += blockDim.x) lsepart[prow0 + static_cast<size_t>(hi) * k] = -INFINITY;
        return;
    }
    const int u0 = j * s, n = min(s, L + 1 - u0);  // keys u0 .. u0+n-1 (causal in the current block)
    for (int e = threadIdx.x; e < G * 128; e += blockDim.x)
        qh[e / 128][e % 128] = __bfloat162float(q[(static_cast<size_t>(bg) * G) * 128 + e]) * scale;
    __syncthreads();
    const __nv_bfloat16 *kr = Kc + (static_cast<size_t>(bg) * T + u0) * 128;
    const __nv_bfloat16 *vr = Vc + (static_cast<size_t>(bg) * T + u0) * 128;
    // scores: warp w takes keys w, w + 8, ...; lane l dims 4l .. 4l+3
    for (int u = warp; u < n; u += kDecThreads / 32) {
        const uint2 kw = __ldg(reinterpret_cast<const uint2 *>(kr + static_cast<size_t>(u) * 128) + lane);
        const float k0 = __uint_as_float(kw.x << 16), k1 = __uint_as_float(kw.x & 0xFFFF0000u);
        const float k2 = __uint_as_float(kw.y << 16), k3 = __uint_as_float(kw.y & 0xFFFF0000u);
        for (int hi = 0; hi < G; ++hi) {
            const float4 qv = reinterpret_cast<const float4 *>(qh[hi])[lane];
            float part = qv.x * k0 + qv.y * k1 + qv.z * k2 + qv.w * k3;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            if (lane == 0) S[hi][u] = part;
        }
    }
    __syncthreads();
    // per head (warp w takes heads w, w + 8): max, weights, sum; then o = sum_u p_u v_u / l
    for (int hi = warp; hi < G; hi += kDecThreads / 32) {
        float m = -INFINITY;
        for (int u = lane; u < n; u += 32) m = fmaxf(m, S[hi][u]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f;
        for (int u = lane; u < n; u += 32) {
            const float p = __expf(S[hi][u] - m);
            S[hi][u] = p;
            l += p;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        __syncwarp();
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int u = 0; u < n; ++u) {
            const uint2 vw = __ldg(reinterpret_cast<const uint2 *>(vr + static_cast<size_t>(u) * 128) + lane);
            const float p = S[hi][u];
            acc[0] = fmaf(p, __uint_as_float(vw.x << 16), acc[0]);
            acc[1] = fmaf(p, __uint_as_float(vw.x & 0xFFFF0000u), acc[1]);
            acc[2] = fmaf(p, __uint_as_float(vw.y << 16), acc[2]);
            acc[3] = fmaf(p, __uint_as_float(vw.y & 0xFFFF0000u), acc[3]);
        }
        const float inv = 1.f / l;
        const size_t pr = prow0 + static_cast<size_t>(hi) * k;
        reinterpret_cast<float4 *>(opart + pr * 128)[lane] =
            make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
        if (lane == 0) lsepart[pr] = m + __logf(l);
    }
}

// One warp per (sequence, query head): o = sum_i exp(lse_i - lse) o_i, lse = log sum_i exp(lse_i).
__global__ void __launch_bounds__(kDecThreads) decode_combine_kernel(const float *__restrict__ opart,
                                                                     const float *__restrict__ lsepart,
                                                                     __nv_bfloat16 *__restrict__ o,
                                                                     float *__restrict__ lse, int nrows, int k) {
    const int row = blockIdx.x * (kDecThreads / 32) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (row >= nrows) return;
    const float *lp = lsepart + static_cast<size_t>(row) * k;
    float mx = -INFINITY;
    for (int i = lane; i < k; i += 32) mx = fmaxf(mx, lp[i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float wsum = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int i = 0; i < k; ++i) {
        const float li = lp[i];
        if (li == -INFINITY) continue;  // unused slot (uniform over the warp)
        const float w = __expf(li - mx);
        wsum += w;
        const float4 v = reinterpret_cast<const float4 *>(opart + (static_cast<size_t>(row) * k + i) * 128)[lane];
        acc[0] = fmaf(w, v.x, acc[0]);
        acc[1] = fmaf(w, v.y, acc[1]);
        acc[2] = fmaf(w, v.z, acc[2]);
        acc[3] = fmaf(w, v.w, acc[3]);
    }
    const float inv = 1.f / wsum;
    reinterpret_cast<uint2 *>(o + static_cast<size_t>(row) * 128)[lane] =
        make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv));
    if (lane == 0) lse[row] = mx + __logf(wsum);
}

}  // namespace ssa
