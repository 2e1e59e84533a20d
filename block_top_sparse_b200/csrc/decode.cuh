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
//   decode_attend_tc_kernel / decode_attend_kernel
//                          one CTA per (sequence, key head, slot): the slot's
//                          block (up to s keys, causal in the current block)
//                          against the G query heads of the group: normalised
//                          partial output and log-sum-exp in fp32 (s = 128:
//                          TMA tiles and tcgen05 MMAs; s = 64: bulk copies and
//                          CUDA-core arithmetic);
//   decode_combine_kernel  one warp per (sequence, query head): log-sum-exp
//                          merge of the k partials.
// Decoding is bound by reading the cache (k*s keys and values and the pooled
// keys of the preceding blocks per key head).
#pragma once

#include "attn_tc.cuh"
#include "pool_select.cuh"

namespace ssa {

constexpr int kDecThreads = 256;
constexpr int kDecMaxBlocks = 1024;  // the warp search holds at most 32 scores per lane
constexpr int kDecMaxGroup = 16;     // query heads per key head

enum : unsigned { ERR_BAD_INPUT = 6u };

// KPL = scores per lane of the warp search: nb <= 32 * KPL.
template <int KPL>
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
    // scores r_j = q . Kbar_j: warp w takes blocks 8w .. 8w+7, then 8w + 64 .., lane l dims 4l .. 4l+3; the
    // eight rows' loads are issued together
    constexpr int R = 8;
    const float4 q4 = reinterpret_cast<const float4 *>(qs)[lane];
    float *kb = Kbar + static_cast<size_t>(bg) * nb * 128;  // this key head's pooled keys
    for (int j0 = R * warp; j0 < bt; j0 += R * (kDecThreads / 32)) {
        float4 v[R];
#pragma unroll
        for (int i = 0; i < R; ++i)
            v[i] = j0 + i < bt ? __ldg(reinterpret_cast<const float4 *>(kb + static_cast<size_t>(j0 + i) * 128) + lane)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
        float mine = 0.f;
#pragma unroll
        for (int i = 0; i < R; ++i) {
            float part = q4.x * v[i].x + q4.y * v[i].y + q4.z * v[i].z + q4.w * v[i].w;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            if (lane == i) mine = part;
        }
        if (lane < R && j0 + lane < bt) sc[j0 + lane] = mine;
    }
    __syncthreads();
    if (warp == 0) select_row<KPL>(sc, bt, min(k - 1, bt), bt, k, out, lane);
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

// Shared memory of decode_attend_kernel<GP>: the slot's keys and values [s][128] bf16 each, bulk-copied
// (reused, once P.V is done, for the eight warps' partial outputs [8][GP][128] fp32); the scores, then
// weights, [s][GP] fp32; per head the max and the sum; two mbarriers and an abort flag.
__host__ __device__ constexpr size_t dec_kv_bytes(int s, int GP) {
    return (static_cast<size_t>(s) * 512 > static_cast<size_t>(GP) * 4096) ? static_cast<size_t>(s) * 512
                                                                            : static_cast<size_t>(GP) * 4096;
}
__host__ __device__ constexpr size_t dec_attend_smem(int s, int GP) {
    return dec_kv_bytes(s, GP) + static_cast<size_t>(s) * GP * 4 + static_cast<size_t>(GP) * 8 + 32;
}

// grid = (B * Hk, k): one slot's block against the group's G query heads (GP = G rounded up to a power of
// two; the padding heads carry a zero query and are not written).
//   1. one thread issues two bulk copies (the block's n <= s key rows, then its value rows, 256 B each), so
//      the whole block is in flight at once; meanwhile every lane loads its four dims of the G query rows;
//   2. scores: a warp takes 32/GP keys at a time, each lane forms the 32 (head, key) partial dot products of
//      its four dims and a transposing butterfly (31 shuffles) leaves lane l with the full sum of pair l;
//   3. a warp per head: max, weights exp(score - max) and their sum;
//   4. P.V: warp w takes the keys [w s/8, (w+1) s/8), each lane four dims of every head; the eight partial
//      outputs are summed through shared memory and normalised: partial output and log-sum-exp in fp32.
template <int GP>
__global__ void __launch_bounds__(kDecThreads) decode_attend_kernel(
    const int32_t *__restrict__ cache_len, const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ Kc,
    const __nv_bfloat16 *__restrict__ Vc, const int32_t *__restrict__ idx, float *__restrict__ opart,
    float *__restrict__ lsepart, int Hk, int G, int T, int s, int k, float scale) {
    extern __shared__ __align__(128) uint8_t dec_att_sm[];
    constexpr int NK = 32 / GP;  // keys per score group: GP heads x NK keys = 32 sums, one per lane
    constexpr int kWarps = kDecThreads / 32;
    const int bg = blockIdx.x, slot = blockIdx.y, b = bg / Hk;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = __ldg(cache_len + b);
    const int j = (L >= 0 && L < T) ? __ldg(idx + static_cast<size_t>(bg) * k + slot) : -1;
    const size_t prow0 = (static_cast<size_t>(bg) * G) * k + slot;  // partial of query head (bg*G + hi): + hi * k
    const size_t kv = dec_kv_bytes(s, GP);
    __nv_bfloat16 *sK = reinterpret_cast<__nv_bfloat16 *>(dec_att_sm);
    __nv_bfloat16 *sV = sK + static_cast<size_t>(s) * 128;
    float *red = reinterpret_cast<float *>(dec_att_sm);     // [8][GP][128], after P.V
    float *P = reinterpret_cast<float *>(dec_att_sm + kv);  // [s][GP]
    float *mx = P + s * GP, *sum = mx + GP;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sum + GP);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 2);
    if (j < 0 || j > L / s) {  // an unused slot (a block past the current one is never selected)
        for (int hi = threadIdx.x; hi < G; hi += blockDim.x) lsepart[prow0 + static_cast<size_t>(hi) * k] = -INFINITY;
        return;
    }
    const int u0 = j * s, n = min(s, L + 1 - u0);  // keys u0 .. u0+n-1 (causal in the current block), n >= 1
    if (threadIdx.x == 0) {
        mbar_init(bars, 1);
        mbar_init(bars + 1, 1);
        *abort_flag = 0;
        fence_barrier_init();
        const uint32_t bytes = static_cast<uint32_t>(n) * 256u;
        const size_t row0 = static_cast<size_t>(bg) * T + u0;
        mbar_arrive_expect_tx(bars, bytes);
        bulk_load(sK, Kc + row0 * 128, bytes, bars);
        mbar_arrive_expect_tx(bars + 1, bytes);
        bulk_load(sV, Vc + row0 * 128, bytes, bars + 1);
    }
    float qv[GP][4];
#pragma unroll
    for (int h = 0; h < GP; ++h) {
        qv[h][0] = qv[h][1] = qv[h][2] = qv[h][3] = 0.f;
        if (h < G) {
            const uint2 w = __ldg(reinterpret_cast<const uint2 *>(q + (static_cast<size_t>(bg) * G + h) * 128) + lane);
            qv[h][0] = __uint_as_float(w.x << 16) * scale;
            qv[h][1] = __uint_as_float(w.x & 0xFFFF0000u) * scale;
            qv[h][2] = __uint_as_float(w.y << 16) * scale;
            qv[h][3] = __uint_as_float(w.y & 0xFFFF0000u) * scale;
        }
    }
    __syncthreads();  // barriers initialised
    if (__syncthreads_or(!mbar_wait(bars, 0, abort_flag, 0x611))) {
        if (threadIdx.x == 0) mbar_drain(bars, 0), mbar_drain(bars + 1, 0);
        return;
    }
    // 2. scores
    const int ng = (n + NK - 1) / NK;
    for (int g = warp; g < ng; g += kWarps) {
        float v[32];
#pragma unroll
        for (int i = 0; i < NK; ++i) {
            const int u = g * NK + i;
            float k0 = 0.f, k1 = 0.f, k2 = 0.f, k3 = 0.f;
            if (u < n) {
                const uint2 kw = *reinterpret_cast<const uint2 *>(sK + u * 128 + 4 * lane);
                k0 = __uint_as_float(kw.x << 16), k1 = __uint_as_float(kw.x & 0xFFFF0000u);
                k2 = __uint_as_float(kw.y << 16), k3 = __uint_as_float(kw.y & 0xFFFF0000u);
            }
#pragma unroll
            for (int h = 0; h < GP; ++h)
                v[h * NK + i] = fmaf(qv[h][0], k0, fmaf(qv[h][1], k1, fmaf(qv[h][2], k2, qv[h][3] * k3)));
        }
        // butterfly: at step `off` a lane keeps the half of its values whose index has bit `off` equal to its
        // own lane bit and adds the partner's copy of that half; after five steps lane l holds sum l.
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            const bool up = (lane & off) != 0;
#pragma unroll
            for (int i = 0; i < off; ++i) {
                const float send = up ? v[i] : v[i + off];
                const float keep = up ? v[i + off] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
            }
        }
        const int u = g * NK + lane % NK;
        if (u < n) P[u * GP + lane / NK] = v[0];
    }
    __syncthreads();
    // 3. softmax numerators per head
    for (int h = warp; h < G; h += kWarps) {
        float m = -INFINITY;
        for (int u = lane; u < n; u += 32) m = fmaxf(m, P[u * GP + h]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f;
        for (int u = lane; u < n; u += 32) {
            const float p = __expf(P[u * GP + h] - m);
            P[u * GP + h] = p;
            l += p;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (lane == 0) mx[h] = m, sum[h] = l;
    }
    if (__syncthreads_or(!mbar_wait(bars + 1, 0, abort_flag, 0x612))) {
        if (threadIdx.x == 0) mbar_drain(bars + 1, 0);
        return;
    }
    // 4. P.V over this warp's keys
    float acc[GP][4];
#pragma unroll
    for (int h = 0; h < GP; ++h) acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
    const int per = s / kWarps, ue = min(n, (warp + 1) * per);
#pragma unroll 4
    for (int u = warp * per; u < ue; ++u) {
        const uint2 vw = *reinterpret_cast<const uint2 *>(sV + u * 128 + 4 * lane);
        const float v0 = __uint_as_float(vw.x << 16), v1 = __uint_as_float(vw.x & 0xFFFF0000u);
        const float v2 = __uint_as_float(vw.y << 16), v3 = __uint_as_float(vw.y & 0xFFFF0000u);
        float p[GP];
        if constexpr (GP >= 4) {
#pragma unroll
            for (int c = 0; c < GP / 4; ++c) {
                const float4 p4 = reinterpret_cast<const float4 *>(P + u * GP)[c];
                p[4 * c] = p4.x, p[4 * c + 1] = p4.y, p[4 * c + 2] = p4.z, p[4 * c + 3] = p4.w;
            }
        } else {
#pragma unroll
            for (int h = 0; h < GP; ++h) p[h] = P[u * GP + h];
        }
#pragma unroll
        for (int h = 0; h < GP; ++h) {
            acc[h][0] = fmaf(p[h], v0, acc[h][0]);
            acc[h][1] = fmaf(p[h], v1, acc[h][1]);
            acc[h][2] = fmaf(p[h], v2, acc[h][2]);
            acc[h][3] = fmaf(p[h], v3, acc[h][3]);
        }
    }
    __syncthreads();  // keys and values are no longer read: their space takes the partial outputs
#pragma unroll
    for (int h = 0; h < GP; ++h)
        reinterpret_cast<float4 *>(red + (warp * GP + h) * 128)[lane] =
            make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
    __syncthreads();
    for (int e = threadIdx.x; e < G * 32; e += kDecThreads) {
        const int h = e >> 5, c4 = e & 31;
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float4 r = reinterpret_cast<const float4 *>(red + (w * GP + h) * 128)[c4];
            o.x += r.x, o.y += r.y, o.z += r.z, o.w += r.w;
        }
        const float inv = 1.f / sum[h];
        const size_t pr = prow0 + static_cast<size_t>(h) * k;
        reinterpret_cast<float4 *>(opart + pr * 128)[c4] = make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
        if (c4 == 0) lsepart[pr] = mx[h] + __logf(sum[h]);
    }
}

// ---------------------------------------------------------------------------
// Tensor-core attend for blocks of s = 128 keys: one CTA (4 warps) per (sequence, key head, slot).
//   the block's keys arrive by TMA (two 64-column chunks, 128-byte swizzle); the group's G query rows
//   (zero-padded to 16) are written into the same layout;
//   S^T [128 keys x 16 heads] = K Q^T  (tcgen05, M = 128, N = 16, K = d; tensor-memory columns 0-15);
//   once that MMA has read the keys, the block's values are loaded by TMA into the same 32 KB, in
//   flight during the softmax;
//   a thread per key: scores of its row (scaled to log2 units, masked past the causal end), maxima
//   and sums per head across the four warps, weights exp2(s - m) as bf16 into the K-major B operand
//   P [16 heads x 128 keys] (the key rows past the causal end hold whatever the cache holds there:
//   their value rows are zeroed so that 0-weighted rows contribute exactly 0);
//   O^T [128 dims x 16 heads] = V^T P^T  (A = V MN-major, columns 16-31);
//   a thread per dim: normalised partial output of each head and its log-sum-exp.
// A CTA's work after its loads land is a chain of dependent steps (MMA, softmax, MMA, output) during
// which it has nothing in flight; keys and values sharing one buffer keep the footprint at ~42 KB, so
// that five CTAs per SM keep enough loads in flight while others run their chains.
// ---------------------------------------------------------------------------
constexpr int kDecTcHeads = 16;  // N of both products

struct DecTcSmem {
    static constexpr int kKV = 0;                         // [2 chunks][128 keys][128 B]: keys, then values
    static constexpr int kQ = kKV + 2 * kChunkBytes;      // [2 chunks][16 heads][128 B]
    static constexpr int kP = kQ + 2 * kDecTcHeads * 128;  // [2 chunks][16 heads][128 B]
    static constexpr int kRed = kP + 2 * kDecTcHeads * 128;  // [2][4 warps][16 heads] fp32: maxima, sums
    static constexpr int kBar = kRed + 2 * 4 * kDecTcHeads * 4;
    static constexpr int kTotal = kBar + 64 + 1024;  // + alignment of the dynamic base to 1024 B
};

__global__ void __launch_bounds__(128) decode_attend_tc_kernel(
    const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
    const int32_t *__restrict__ cache_len, const __nv_bfloat16 *__restrict__ q, const int32_t *__restrict__ idx,
    float *__restrict__ opart, float *__restrict__ lsepart, int Hk, int G, int T, int k, float scale_log2) {
    constexpr int s = 128;
    constexpr int NH = kDecTcHeads;
    constexpr int kHeadChunk = NH * 128;  // bytes of one 64-column chunk of the Q / P operands
    extern __shared__ __align__(1024) uint8_t dtc_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dtc_raw) + 1023) & ~uintptr_t(1023));
    const int bg = blockIdx.x, slot = blockIdx.y, b = bg / Hk;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = __ldg(cache_len + b);
    const int j = (L >= 0 && L < T) ? __ldg(idx + static_cast<size_t>(bg) * k + slot) : -1;
    const size_t prow0 = (static_cast<size_t>(bg) * G) * k + slot;  // partial of query head (bg*G + h): + h * k
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + DecTcSmem::kBar);
    uint64_t *bar_k = bars, *bar_v = bars + 1, *bar_s = bars + 2, *bar_o = bars + 3;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 5);
    if (j < 0 || j > L / s) {  // an unused slot
        for (int h = threadIdx.x; h < G; h += blockDim.x) lsepart[prow0 + static_cast<size_t>(h) * k] = -INFINITY;
        return;
    }
    const int u0 = j * s, n = min(s, L + 1 - u0);  // keys u0 .. u0+n-1, n >= 1
    float *red_m = reinterpret_cast<float *>(smem + DecTcSmem::kRed), *red_l = red_m + 4 * NH;
    const uint32_t sKV = smem_u32(smem + DecTcSmem::kKV);
    const uint32_t sQ = smem_u32(smem + DecTcSmem::kQ), sP = smem_u32(smem + DecTcSmem::kP);
    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(bars + i, 1);
        *abort_flag = 0;
        fence_barrier_init();
        const int row0 = bg * T + u0;  // key/value row of the block's first key (the host keeps B*Hkv*T < 2^31)
        mbar_arrive_expect_tx(bar_k, 2 * kChunkBytes);
        tma_load_2d(&mapK, bar_k, smem + DecTcSmem::kKV, 0, row0);
        tma_load_2d(&mapK, bar_k, smem + DecTcSmem::kKV + kChunkBytes, 64, row0);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 32);
        tmem_relinquish();
    }
    // the group's query rows as the K-major B operand: row h (zero past G), 16-byte unit c of a 64-column
    // chunk stored at unit c ^ (h & 7)
    for (int e = threadIdx.x; e < 2 * NH * 8; e += blockDim.x) {
        const int c2 = e / (NH * 8), h = (e / 8) % NH, c = e % 8;
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (h < G)
            w = __ldg(reinterpret_cast<const uint4 *>(q + (static_cast<size_t>(bg) * G + h) * 128 + c2 * 64 + c * 8));
        *reinterpret_cast<uint4 *>(smem + DecTcSmem::kQ + c2 * kHeadChunk + h * 128 + ((c ^ (h & 7)) << 4)) = w;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;  // S^T: columns 0-15, O^T: columns 16-31
    bool issued_s = false, issued_v = false, issued_o = false;  // (thread 0)
    // exit path on a wait that gave up: let this CTA's loads and MMAs in flight finish, free the columns
    auto give_up = [&]() {
        if (threadIdx.x == 0) {
            mbar_drain(bar_k, 0);
            if (issued_v) mbar_drain(bar_v, 0);
            if (issued_s) mbar_drain(bar_s, 0);
            if (issued_o) mbar_drain(bar_o, 0);
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (warp == 1) tmem_dealloc(tmem, 32);
    };
    if (threadIdx.x == 0 && mbar_wait(bar_k, 0, abort_flag, 0x621)) {
        tc_fence_after();
        mma_k128_kmajor(tmem, sKV, sQ, kHeadChunk, idesc_bf16(128, NH, false, false));
        mma_commit(bar_s);
        issued_s = true;
        if (mbar_wait(bar_s, 0, abort_flag, 0x625)) {  // the keys have been read: values into their space
            const int row0 = bg * T + u0;
            mbar_arrive_expect_tx(bar_v, 2 * kChunkBytes);
            tma_load_2d(&mapV, bar_v, smem + DecTcSmem::kKV, 0, row0);
            tma_load_2d(&mapV, bar_v, smem + DecTcSmem::kKV + kChunkBytes, 64, row0);
            issued_v = true;
        }
    }
    if (__syncthreads_or(!mbar_wait(bar_s, 0, abort_flag, 0x622))) {
        give_up();
        return;
    }
    tc_fence_after();
    const int u = warp * 32 + lane;  // this thread's key
    const bool valid = u < n;
    float sc[NH];
    tmem_ld16(tmem + (static_cast<uint32_t>(warp * 32) << 16), sc);
#pragma unroll
    for (int h = 0; h < NH; ++h) {
        if (h < G) {
            sc[h] = valid ? sc[h] * scale_log2 : -INFINITY;
            float m = sc[h];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) red_m[warp * NH + h] = m;
        }
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < NH; ++h) {
        if (h < G) {
            const float m = fmaxf(fmaxf(red_m[h], red_m[NH + h]), fmaxf(red_m[2 * NH + h], red_m[3 * NH + h]));
            sc[h] = valid ? fast_exp2(sc[h] - m) : 0.f;
            float l = sc[h];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
            if (lane == 0) red_l[warp * NH + h] = l;
        }
    }
    if (__syncthreads_or(!mbar_wait(bar_v, 0, abort_flag, 0x623))) {
        give_up();
        return;
    }
    if (!valid) {  // a key past the causal end: zero its value row (both chunks; the swizzle stays inside a row)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            *reinterpret_cast<uint4 *>(smem + DecTcSmem::kKV + u * 128 + c * 16) = make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4 *>(smem + DecTcSmem::kKV + kChunkBytes + u * 128 + c * 16) =
                make_uint4(0u, 0u, 0u, 0u);
        }
    }
    {  // weights as the K-major B operand: row h, key u in chunk u / 64, unit ((u % 64) / 8) ^ (h & 7)
        const int c2 = u >> 6, uu = u & 63;
        uint8_t *prow = smem + DecTcSmem::kP + c2 * kHeadChunk + (uu & 7) * 2;
#pragma unroll
        for (int h = 0; h < NH; ++h)
            if (h < G)
                *reinterpret_cast<__nv_bfloat16 *>(prow + h * 128 + (((uu >> 3) ^ (h & 7)) << 4)) =
                    __float2bfloat16_rn(sc[h]);
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) {
        tc_fence_after();
        const uint32_t idO = idesc_bf16(128, NH, true, false);
#pragma unroll
        for (int kk = 0; kk < s / 16; ++kk)
            mma_bf16_ss(tmem + 16, smem_desc_sw128(sKV + kk * 2048, kChunkBytes),
                        smem_desc_sw128(sP + (kk >> 2) * kHeadChunk + (kk & 3) * 32, 16), idO, kk > 0 ? 1u : 0u);
        mma_commit(bar_o);
        issued_o = true;
    }
    if (__syncthreads_or(!mbar_wait(bar_o, 0, abort_flag, 0x624))) {
        give_up();
        return;
    }
    tc_fence_after();
    float ot[NH];
    tmem_ld16(tmem + 16 + (static_cast<uint32_t>(warp * 32) << 16), ot);  // lane = dim
    const int dcol = warp * 32 + lane;
#pragma unroll
    for (int h = 0; h < NH; ++h) {
        if (h < G) {
            const float l = red_l[h] + red_l[NH + h] + red_l[2 * NH + h] + red_l[3 * NH + h];
            opart[(prow0 + static_cast<size_t>(h) * k) * 128 + dcol] = ot[h] / l;
        }
    }
    if (threadIdx.x < G) {
        const int h = threadIdx.x;
        const float m = fmaxf(fmaxf(red_m[h], red_m[NH + h]), fmaxf(red_m[2 * NH + h], red_m[3 * NH + h]));
        const float l = red_l[h] + red_l[NH + h] + red_l[2 * NH + h] + red_l[3 * NH + h];
        lsepart[prow0 + static_cast<size_t>(h) * k] = (m + __log2f(l)) * 0.69314718055994531f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 32);
}

// One warp per (sequence, query head): o = sum_i exp(lse_i - lse) o_i, lse = log sum_i exp(lse_i).
__global__ void __launch_bounds__(kDecThreads) decode_combine_kernel(const float *__restrict__ opart,
                                                                     const float *__restrict__ lsepart,
                                                                     __nv_bfloat16 *__restrict__ o,
                                                                     float *__restrict__ lse, int nrows, int k) {
    const int row = blockIdx.x * (kDecThreads / 32) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (row >= nrows) return;
    const float *lp = lsepart + static_cast<size_t>(row) * k;
    const float4 *op = reinterpret_cast<const float4 *>(opart + static_cast<size_t>(row) * k * 128) + lane;
    float mx = -INFINITY;
    for (int i = lane; i < k; i += 32) mx = fmaxf(mx, lp[i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float wsum = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
    // partials 32 at a time: lane i holds the log-sum-exp of partial i0 + i and hands it to the warp by a
    // shuffle, so that the partial outputs' loads depend on no memory read and go out together
    for (int i0 = 0; i0 < k; i0 += 32) {
        const int nk = min(32, k - i0);
        const float mine = lane < nk ? lp[i0 + lane] : -INFINITY;
#pragma unroll 8
        for (int i = 0; i < nk; ++i) {
            const float li = __shfl_sync(0xffffffffu, mine, i);
            // an unused slot (uniform over the warp) has no partial output: weight 0, nothing read
            const float w = li == -INFINITY ? 0.f : __expf(li - mx);
            const float4 v = li == -INFINITY ? make_float4(0.f, 0.f, 0.f, 0.f) : op[static_cast<size_t>(i0 + i) * 32];
            wsum += w;
            acc[0] = fmaf(w, v.x, acc[0]);
            acc[1] = fmaf(w, v.y, acc[1]);
            acc[2] = fmaf(w, v.z, acc[2]);
            acc[3] = fmaf(w, v.w, acc[3]);
        }
    }
    const float inv = 1.f / wsum;
    reinterpret_cast<uint2 *>(o + static_cast<size_t>(row) * 128)[lane] =
        make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv));
    if (lane == 0) lse[row] = mx + __logf(wsum);
}

}  // namespace ssa
