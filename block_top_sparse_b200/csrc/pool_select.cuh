// pool_select.cuh -- block pooling and per-query causal top-k block selection.
//
// Paper section 3: keys are partitioned into contiguous blocks of s tokens,
// each block is mean-pooled, every strictly preceding block is scored against
// the query (r_j = q . Kbar_j) and the top blocks are kept.  Reading used here:
// the query's own block is always kept and counted within k; ties go to the
// lower block index; rows are ascending with -1 padding at the end.
#pragma once

#include "device.cuh"

namespace ssa {

// 16-byte vector load of dtype T converted to fp32.
template <typename T>
struct Vec16;

template <>
struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float (&f)[8]) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};

template <>
struct Vec16<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void load(const float *p, float (&f)[4]) {
        const float4 u = __ldg(reinterpret_cast<const float4 *>(p));
        f[0] = u.x;
        f[1] = u.y;
        f[2] = u.z;
        f[3] = u.w;
    }
};

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}
template <>
__device__ __forceinline__ float to_f32<float>(float x) {
    return x;
}

// ---------------------------------------------------------------------------
// Pooling: one CTA (256 threads) per (head, block).  Thread (row group g,
// column vector c) sums rows g, g+G, ... in order; the G partial sums are then
// added in fixed order and divided by s.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) pool_kernel(const T *__restrict__ K, float *__restrict__ Kbar, int T_len, int d,
                                                   int s, int nb) {
    constexpr int V = Vec16<T>::N;
    __shared__ float part[256 * V];
    const int tpr = d / V;                  // threads per row
    const int G = blockDim.x / tpr;         // rows in flight
    const int g = threadIdx.x / tpr, cv = threadIdx.x % tpr;
    const int bh = blockIdx.x / nb, j = blockIdx.x % nb;
    const T *base = K + (static_cast<size_t>(bh) * T_len + static_cast<size_t>(j) * s) * d + cv * V;
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.f;
#pragma unroll 8
    for (int r = g; r < s; r += G) {
        float f[V];
        Vec16<T>::load(base + static_cast<size_t>(r) * d, f);
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] += f[i];
    }
#pragma unroll
    for (int i = 0; i < V; ++i) part[g * d + cv * V + i] = acc[i];
    __syncthreads();
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        float sum = 0.f;
        for (int q = 0; q < G; ++q) sum += part[q * d + c];
        Kbar[(static_cast<size_t>(bh) * nb + j) * d + c] = sum / static_cast<float>(s);
    }
}

// ---------------------------------------------------------------------------
// Selection.  One CTA (256 threads) per 32 consecutive queries of one head
// (all in the same block, since s is a multiple of 32); warp w owns queries
// 4w .. 4w+3 from scoring to output.
//   scores: r[q][j] = q . Kbar_j for j < b(t), fp32 FMA in column order; Kbar
//           staged 64 blocks at a time; lane l of warp w scores blocks l and
//           l + 32 of the chunk for the warp's 4 queries;
//   top-(k-1): the (k-1)-th largest order-preserving 32-bit key is built bit by
//           bit from the most significant end (count of keys >= candidate by
//           warp reduction), stopping early at a candidate with exactly k-1 keys
//           at or above it; otherwise keys above it are kept, keys equal to it
//           are kept in ascending block order until k-1 are chosen; a ballot compaction
//           writes the chosen blocks in ascending order, then b(t), then -1.
// ---------------------------------------------------------------------------
constexpr int kSelQ = 32;
constexpr int kSelJ = 64;

__host__ __device__ constexpr size_t select_smem_bytes(int d, int nb) {
    return (static_cast<size_t>(kSelQ + kSelJ) * (d + 4) + static_cast<size_t>(kSelQ) * nb) * 4;
}

__device__ __forceinline__ uint32_t order_key(float x) {
    uint32_t u = __float_as_uint(x);
    if (u == 0x80000000u) u = 0u;  // -0 ranks as +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-(want) of row[0..n) for one warp; KPL keys per lane (n <= 32*KPL).
// Invariant of the search: at least `want` keys are >= tau.  A candidate with exactly
// `want` keys at or above it separates the top `want` from the rest: stop there (no key
// equal to the threshold is left out); otherwise tau ends as the want-th largest key and
// need_eq of the keys equal to it are taken in ascending block order.
struct SelSearch {
    uint32_t tau = 0u;
    int need_eq = 0;
    bool exact = false;
    bool done = true;
};

template <int KPL>
__device__ __forceinline__ void select_load(const float *row, int n, uint32_t (&key)[KPL], int lane) {
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
        const int j = 32 * i + lane;
        key[i] = j < n ? order_key(row[j]) : 0u;  // 0 is below every real key
    }
}

template <int KPL>
__device__ __forceinline__ unsigned select_count(const uint32_t (&key)[KPL], uint32_t cand) {
    unsigned c = 0;
#pragma unroll
    for (int i = 0; i < KPL; ++i) c += key[i] >= cand ? 1u : 0u;
    return __reduce_add_sync(0xffffffffu, c);
}

// One step (bit b) of the search; a finished search is left unchanged.
__device__ __forceinline__ void select_step(SelSearch &st, int want, int b, unsigned tot) {
    if (st.done) return;
    if (tot >= static_cast<unsigned>(want)) {
        st.tau |= 1u << b;
        if (tot == static_cast<unsigned>(want)) {
            st.exact = true;
            st.done = true;
        }
    }
}

template <int KPL>
__device__ __forceinline__ void select_finish(const uint32_t (&key)[KPL], SelSearch &st, int want, int n) {
    if (want > 0 && want < n && !st.exact) {
        unsigned gt = 0;
#pragma unroll
        for (int i = 0; i < KPL; ++i) gt += key[i] > st.tau ? 1u : 0u;
        st.need_eq = want - static_cast<int>(__reduce_add_sync(0xffffffffu, gt));
    }
}

// Writes the chosen blocks ascending, then b(t), then -1 padding up to k.
template <int KPL>
__device__ __forceinline__ void select_emit(const uint32_t (&key)[KPL], const SelSearch &st, int n, int want, int bt,
                                            int k, int32_t *out, int lane) {
    const uint32_t lt_mask = (1u << lane) - 1u;
    int taken = 0, eq_seen = 0;
    if (want > 0) {
#pragma unroll
        for (int i = 0; i < KPL; ++i) {
            if (32 * i >= n) break;
            const bool in = 32 * i + lane < n;
            bool sel;
            uint32_t eqb = 0u;
            if (want < n && st.exact) {
                sel = in && key[i] >= st.tau;
            } else if (want < n) {
                const bool eq = in && key[i] == st.tau;
                eqb = __ballot_sync(0xffffffffu, eq);
                sel = (in && key[i] > st.tau) || (eq && (eq_seen + __popc(eqb & lt_mask)) < st.need_eq);
            } else {
                sel = in;
            }
            const uint32_t sb = __ballot_sync(0xffffffffu, sel);
            const int pos = taken + __popc(sb & lt_mask);
            if (sel && pos < want) out[pos] = 32 * i + lane;
            taken += __popc(sb);
            eq_seen += __popc(eqb);
        }
    }
    for (int i = want + lane; i < k; i += 32) out[i] = (i == want) ? bt : -1;
}

template <int KPL>
__device__ __forceinline__ void select_row(const float *row, int n, int want, int bt, int k, int32_t *out, int lane) {
    uint32_t key[KPL];
    select_load<KPL>(row, n, key, lane);
    SelSearch st;
    st.done = !(want > 0 && want < n);
#pragma unroll 1
    for (int b = 31; b >= 0 && !st.done; --b) select_step(st, want, b, select_count<KPL>(key, st.tau | (1u << b)));
    select_finish<KPL>(key, st, want, n);
    select_emit<KPL>(key, st, n, want, bt, k, out, lane);
}

// Two rows' searches interleaved in one warp: their chains of dependent warp reductions overlap.
template <int KPL>
__device__ __forceinline__ void select_row2(const float *rowA, int nA, int wantA, int btA, int32_t *outA,
                                            const float *rowB, int nB, int wantB, int btB, int32_t *outB, int k,
                                            int lane) {
    uint32_t ka[KPL], kb[KPL];
    select_load<KPL>(rowA, nA, ka, lane);
    select_load<KPL>(rowB, nB, kb, lane);
    SelSearch sa, sb;
    sa.done = !(wantA > 0 && wantA < nA);
    sb.done = !(wantB > 0 && wantB < nB);
#pragma unroll 1
    for (int b = 31; b >= 0 && !(sa.done && sb.done); --b) {
        const unsigned ta = select_count<KPL>(ka, sa.tau | (1u << b));
        const unsigned tb = select_count<KPL>(kb, sb.tau | (1u << b));
        select_step(sa, wantA, b, ta);
        select_step(sb, wantB, b, tb);
    }
    select_finish<KPL>(ka, sa, wantA, nA);
    select_finish<KPL>(kb, sb, wantB, nB);
    if (outA) select_emit<KPL>(ka, sa, nA, wantA, btA, k, outA, lane);
    if (outB) select_emit<KPL>(kb, sb, nB, wantB, btB, k, outB, lane);
}

template <typename T, int KPL>
__global__ void __launch_bounds__(256) select_kernel(const T *__restrict__ Q, const float *__restrict__ Kbar,
                                                     int32_t *__restrict__ idx, int T_len, int d, int s, int k,
                                                     int nb) {
    extern __shared__ __align__(16) float sm[];
    const int dp = d + 4;
    float *sQ = sm;                       // [32][dp]
    float *sK = sQ + kSelQ * dp;          // [64][dp]
    float *sS = sK + kSelJ * dp;          // [32][nb]

    const int bh = blockIdx.y, t0 = blockIdx.x * kSelQ;
    const int bt = t0 / s;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    for (int e = tid; e < kSelQ * d; e += blockDim.x) {
        const int qi = e / d, c = e % d;
        sQ[qi * dp + c] = to_f32(Q[(static_cast<size_t>(bh) * T_len + t0 + qi) * d + c]);
    }
    for (int jc = 0; jc < bt; jc += kSelJ) {
        const int nj = min(kSelJ, bt - jc);
        __syncthreads();
        for (int e = tid; e < nj * (d / 4); e += blockDim.x) {
            const int jj = e / (d / 4), c4 = e % (d / 4);
            *reinterpret_cast<float4 *>(sK + jj * dp + c4 * 4) =
                __ldg(reinterpret_cast<const float4 *>(Kbar + (static_cast<size_t>(bh) * nb + jc + jj) * d) + c4);
        }
        __syncthreads();
        float acc[4][2];
#pragma unroll
        for (int a = 0; a < 4; ++a) acc[a][0] = acc[a][1] = 0.f;
#pragma unroll 4
        for (int c = 0; c < d; c += 4) {
            float4 qv[4], kv[2];
#pragma unroll
            for (int a = 0; a < 4; ++a) qv[a] = *reinterpret_cast<const float4 *>(sQ + (4 * warp + a) * dp + c);
#pragma unroll
            for (int b = 0; b < 2; ++b) kv[b] = *reinterpret_cast<const float4 *>(sK + (lane + 32 * b) * dp + c);
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    acc[a][b] = fmaf(qv[a].x, kv[b].x, acc[a][b]);
                    acc[a][b] = fmaf(qv[a].y, kv[b].y, acc[a][b]);
                    acc[a][b] = fmaf(qv[a].z, kv[b].z, acc[a][b]);
                    acc[a][b] = fmaf(qv[a].w, kv[b].w, acc[a][b]);
                }
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                const int jj = lane + 32 * b;
                if (jj < nj) sS[(4 * warp + a) * nb + jc + jj] = acc[a][b];
            }
    }
    __syncwarp();
    const int want = min(k - 1, bt);
    for (int qq = 0; qq < 4; ++qq) {
        const int qi = 4 * warp + qq;
        select_row<KPL>(sS + qi * nb, bt, want, bt, k, idx + (static_cast<size_t>(bh) * T_len + t0 + qi) * k, lane);
    }
}

// ---------------------------------------------------------------------------
// Selection with the block scores on the tensor cores (bf16 Q, d = 128, nb <= 256).
// One CTA (512 threads) per 128 consecutive queries of one head:
//   scores: r[q][j] = q . Kbar_j as one dense contraction S = Q Kbar^T (M = 128 queries,
//           N = 64 blocks per group, K = d) in tensor memory.  Kbar (fp32) is split into
//           three bf16 terms, hi = bf16(x), mid = bf16(x - hi), lo = bf16(x - hi - mid),
//           which carry its 24 significant bits; the products with the bf16 query are
//           exact and the three contractions accumulate in fp32;
//   top-(k-1): the scores are staged row-major in shared memory and each of the 16 warps runs
//           the threshold search of select_row on 8 of the 128 rows (a search is a chain of
//           dependent warp reductions, so many rows are kept in flight).
// ---------------------------------------------------------------------------
constexpr int kSelTcRows = 128;
constexpr int kSelTcThreads = 512;
constexpr int kSelTcWarps = kSelTcThreads / 32;
constexpr int kSelTcMaxBlocks = 256;
constexpr int kSelTcPitch = kSelTcMaxBlocks + 4;  // fp32 score row pitch: conflict-free staging

struct SelTcSmem {
    static constexpr int kQ = 0;                      // 128 rows x 128 bf16: 2 swizzled 16 KB chunks
    static constexpr int kB = 2 * 16384;              // hi / mid / lo: 3 x (64 blocks x 128 bf16), 16 KB each
    static constexpr int kS = kB + 3 * 16384;         // 128 x kSelTcPitch fp32 scores
    static constexpr int kBar = kS + kSelTcRows * kSelTcPitch * 4;
    static constexpr int kTotal = kBar + 64;
};

__device__ __forceinline__ void st_shared_v2(uint32_t addr, uint32_t a, uint32_t b) {
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}

__global__ void __launch_bounds__(kSelTcThreads, 1) select_tc_kernel(const __nv_bfloat16 *__restrict__ Q,
                                                           const float *__restrict__ Kbar, int32_t *__restrict__ idx,
                                                           int T_len, int s, int k, int nb) {
    using L = SelTcSmem;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar_mma = reinterpret_cast<uint64_t *>(smem + L::kBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kBar + 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kBar + 16);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.y, t0 = blockIdx.x * kSelTcRows;
    const size_t head_rows = static_cast<size_t>(bh) * T_len;
    const int last = min(t0 + kSelTcRows, T_len) - 1;
    const int nbc = min(last / s, nb);  // blocks scored by some row of the tile (j < b(t))
    const int ngroups = (nbc + 63) / 64;
    const uint32_t sQ = smem_u32(smem + L::kQ), sB = smem_u32(smem + L::kB);
    float *sS = reinterpret_cast<float *>(smem + L::kS);

    if (tid == 0) {
        mbar_init(bar_mma, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    {
        // query rows -> K-major 128-byte-swizzled tile; rows past T are zero-filled
        const int u = tid & 15;
        for (int row = tid >> 4; row < kSelTcRows; row += kSelTcThreads / 16) {
            const int t = t0 + row;
            const bool valid = t < T_len;
            const uint32_t dst = sQ + (u >> 3) * 16384 + row * 128 + ((((u & 7) ^ (row & 7)) & 7) << 4);
            cp_async_16(dst, Q + (head_rows + (valid ? t : 0)) * 128 + u * 8, valid ? 16u : 0u);
        }
        cp_async_wait_all();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;
    for (int gi = 0; gi < ngroups; ++gi) {
        // Kbar rows 64gi .. 64gi+63 -> hi / mid / lo tiles (K-major, swizzled); rows >= nbc are zero.
        // Lane c4 of a warp takes dims 4c4 .. 4c4+3 of one row: two 128-byte row halves per store.
        const int c4 = lane;
        for (int jj = warp; jj < 64; jj += kSelTcWarps) {
            const int j = 64 * gi + jj;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (j < nbc) v = __ldg(reinterpret_cast<const float4 *>(Kbar + (static_cast<size_t>(bh) * nb + j) * 128) + c4);
            const uint32_t h01 = pack_bf16x2(v.x, v.y), h23 = pack_bf16x2(v.z, v.w);
            const float r0 = v.x - __uint_as_float(h01 << 16), r1 = v.y - __uint_as_float(h01 & 0xFFFF0000u);
            const float r2 = v.z - __uint_as_float(h23 << 16), r3 = v.w - __uint_as_float(h23 & 0xFFFF0000u);
            const uint32_t m01 = pack_bf16x2(r0, r1), m23 = pack_bf16x2(r2, r3);
            const uint32_t l01 = pack_bf16x2(r0 - __uint_as_float(m01 << 16), r1 - __uint_as_float(m01 & 0xFFFF0000u));
            const uint32_t l23 = pack_bf16x2(r2 - __uint_as_float(m23 << 16), r3 - __uint_as_float(m23 & 0xFFFF0000u));
            const uint32_t off = (c4 >> 4) * 8192 + jj * 128 + (((((c4 & 15) >> 1) ^ (jj & 7)) & 7) << 4) + (c4 & 1) * 8;
            st_shared_v2(sB + off, h01, h23);
            st_shared_v2(sB + 16384 + off, m01, m23);
            st_shared_v2(sB + 2 * 16384 + off, l01, l23);
        }
        fence_proxy_async_smem();  // generic-proxy tile writes -> tensor-core reads
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int sp = 0; sp < 3; ++sp)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ss(tmem + 64 * gi, smem_desc_sw128(sQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16),
                                smem_desc_sw128(sB + sp * 16384 + (kk >> 2) * 8192 + (kk & 3) * 32, 16), id,
                                (sp > 0 || kk > 0) ? 1u : 0u);
            mma_commit(bar_mma);
        }
        // the next group rewrites the split tiles only after these MMAs have read them
        if (!mbar_wait(bar_mma, gi & 1, abort_flag, 0x501)) {
            ok = false;
            break;
        }
    }
    tc_fence_after();
    // scores -> shared memory: warps 0-3, thread <-> row (tensor-memory lane)
    if (ok && warp < 4) {
        const int row = warp * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t dst = smem_u32(sS + row * kSelTcPitch);
        for (int c = 0; c < 2 * ngroups; ++c) {
            uint32_t v[32];
            tmem_ld32_async(tmem + lane_off + 32 * c, v);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 8; ++q) st_shared_v4(dst + (32 * c + 4 * q) * 4, v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 256);
    // top-(k-1) per row: warp w takes rows w, w + 16, ..., two at a time (rows past T write nothing)
    for (int row = warp; row < kSelTcRows; row += 2 * kSelTcWarps) {
        const int ta = t0 + row, tb = t0 + row + kSelTcWarps;
        const int bta = ta / s, btb = tb / s;
        const bool va = ta < T_len, vb = tb < T_len;
        select_row2<8>(sS + row * kSelTcPitch, va ? bta : 0, va ? min(k - 1, bta) : 0, bta,
                       va ? idx + (head_rows + ta) * k : nullptr, sS + (row + kSelTcWarps) * kSelTcPitch,
                       vb ? btb : 0, vb ? min(k - 1, btb) : 0, btb, vb ? idx + (head_rows + tb) * k : nullptr, k,
                       lane);
    }
}

}  // namespace ssa
