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
// Pooling: one warp per (head, block), no shared memory and no CTA barrier.
// A warp instruction reads 512 contiguous bytes: lane l takes the 16-byte unit
// l % U of row l / U (U = units per row, R = 32 / U rows per instruction), so
// every load of the block is a full coalesced line set.  Each lane keeps
// kPoolInFlight loads in flight, sums its unit's columns in fp32 over the rows
// it visits (in row order), and the R lanes that hold the same columns are
// combined by shuffles; lanes of row slot 0 write Kbar = sum / s.
// ---------------------------------------------------------------------------
constexpr int kPoolWarps = 8;     // warps (blocks) per CTA
constexpr int kPoolInFlight = 16;  // 16-byte loads in flight per lane (one pass covers R * 16 <= 64 rows)

template <typename T, int D>
__global__ void __launch_bounds__(kPoolWarps * 32) pool_kernel(const T *__restrict__ K, float *__restrict__ Kbar,
                                                             int T_len, int s, int nb, size_t units) {
    constexpr int V = Vec16<T>::N;      // elements per 16-byte unit
    constexpr int U = D / V;            // units per row
    constexpr int R = 32 / U;           // rows per warp instruction
    const int lane = threadIdx.x & 31;
    const size_t u = static_cast<size_t>(blockIdx.x) * kPoolWarps + (threadIdx.x >> 5);
    if (u >= units) return;
    const size_t bh = u / nb;
    const int j = static_cast<int>(u % nb);
    const int cu = lane % U, ro = lane / U;
    const T *base = K + (bh * T_len + static_cast<size_t>(j) * s) * D + cu * V;
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.f;
    for (int r0 = 0; r0 < s; r0 += R * kPoolInFlight) {
        // all the raw 16-byte units first (kPoolInFlight loads in flight), then the fp32 sums
        // (s in {64, 128} is a multiple of the R * kPoolInFlight <= 64 rows of one pass)
        uint4 raw[kPoolInFlight];
#pragma unroll
        for (int q = 0; q < kPoolInFlight; ++q)
            raw[q] = __ldg(reinterpret_cast<const uint4 *>(base + static_cast<size_t>(r0 + q * R + ro) * D));
#pragma unroll
        for (int q = 0; q < kPoolInFlight; ++q) {
            const uint32_t w[4] = {raw[q].x, raw[q].y, raw[q].z, raw[q].w};
            if constexpr (sizeof(T) == 2) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    acc[2 * i] += __uint_as_float(w[i] << 16);
                    acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[i] += __uint_as_float(w[i]);
            }
        }
    }
    // lanes ro = 0 .. R-1 of the same unit hold partial sums of the same columns
#pragma unroll
    for (int o = U; o < 32; o <<= 1)
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
    if (ro == 0) {
        const float inv = 1.f / static_cast<float>(s);
        float4 *dst = reinterpret_cast<float4 *>(Kbar + u * D + cu * V);
#pragma unroll
        for (int i = 0; i < V; i += 4)
            dst[i / 4] = make_float4(acc[i] * inv, acc[i + 1] * inv, acc[i + 2] * inv, acc[i + 3] * inv);
    }
}

// ---------------------------------------------------------------------------
// Selection.  One CTA (256 threads) per 32 consecutive queries of one key/value
// head (all in the same block, since s is a multiple of 32); warp w owns queries
// 4w .. 4w+3 from scoring to output.  With G query heads per key head the query
// row scored is the fp32 sum of the group's rows (the sum of the heads' scores up
// to fp32 rounding).
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

template <typename T, int KPL>
__global__ void __launch_bounds__(256) select_kernel(const T *__restrict__ Q, const float *__restrict__ Kbar,
                                                     int32_t *__restrict__ idx, int T_len, int d, int s, int k,
                                                     int nb, int G) {
    extern __shared__ __align__(16) float sm[];
    const int dp = d + 4;
    float *sQ = sm;                       // [32][dp]
    float *sK = sQ + kSelQ * dp;          // [64][dp]
    float *sS = sK + kSelJ * dp;          // [32][nb]

    const int bh = blockIdx.y, t0 = blockIdx.x * kSelQ;
    const int bt = t0 / s;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // the query row of the group: the fp32 sum of its G heads' rows (G = 1: the row itself)
    for (int e = tid; e < kSelQ * d; e += blockDim.x) {
        const int qi = e / d, c = e % d;
        float v = 0.f;
        for (int hi = 0; hi < G; ++hi)
            v += to_f32(Q[((static_cast<size_t>(bh) * G + hi) * T_len + t0 + qi) * d + c]);
        sQ[qi * dp + c] = v;
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
//           N = 64 blocks per group, K = d) in tensor memory; with G query heads per key
//           head, the G heads' contractions accumulate into the same scores (the group's
//           selection ranks by the sum of its heads' scores).  Kbar (fp32) is split into
//           three bf16 terms, hi = bf16(x), mid = bf16(x - hi), lo = bf16(x - hi - mid),
//           which carry its 24 significant bits; the products with the bf16 query are
//           exact and the three contractions accumulate in fp32;
//   top-(k-1): thread <-> query row (tensor-memory lane).  Warp w reads rows
//           32 (w & 3) .. +31 and the 32-column chunks c = w >> 2, (w >> 2) + 4 of the
//           scores straight from tensor memory into registers (64 per thread at most), so
//           the four warps of a row group share each row's candidates.  The (k-1)-th
//           largest order key tau is built bit by bit from the most significant end: each
//           step counts, per row, the scores at or above the candidate threshold (compared
//           as floats against the threshold's value), and the four partial counts meet in
//           shared memory behind one named barrier of the row group; the search stops at a
//           threshold with exactly k-1 scores at or above it.  Otherwise the scores above
//           tau are kept and those equal to it in ascending block order until k-1 are
//           chosen (lowest index wins ties).  Each warp then leaves the chosen columns of
//           its chunks as 32-bit masks, and one warp per row group writes the row:
//           chosen blocks ascending, b(t), -1 padding.
// ---------------------------------------------------------------------------
constexpr int kSelTcRows = 128;
constexpr int kSelTcThreads = 512;
constexpr int kSelTcMaxBlocks = 256;

constexpr int kSelList = 16;  // register top list per thread (k - 1 <= kSelList)

struct SelTcSmem {
    static constexpr int kQ = 0;                      // 128 rows x 128 bf16: 2 swizzled 16 KB chunks
    static constexpr int kB = 2 * 16384;              // [2 buffers] hi / mid / lo: 3 x (64 blocks x 128 bf16)
    static constexpr int kBBuf = 3 * 16384;
    static constexpr int kCnt = kB + 2 * kBBuf;       // [2 steps][4 column groups][128 rows] partial counts
    static constexpr int kMask = kCnt + 2 * 4 * 128 * 4;  // [8 chunks][128 rows] x {above, equal} masks
    static constexpr int kList = kMask + 2 * 8 * 128 * 4;  // [4 column groups][128 rows][kSelList] top lists
    static constexpr int kThr = kList + 4 * 128 * kSelList * 4;  // [128 rows] thresholds
    static constexpr int kBar = kThr + 128 * 4;
    static constexpr int kTotal = kBar + 64;
};

__device__ __forceinline__ void st_shared_v2(uint32_t addr, uint32_t a, uint32_t b) {
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}

// The float whose order key is `key` (inverse of order_key): key(x) >= key <=> x >= value, for every
// non-NaN x.  Keys above that of +inf map to NaN (nothing compares at or above them); keys at or below
// that of -inf map to -inf (everything does).
__device__ __forceinline__ float key_value(uint32_t key) {
    if (key & 0x80000000u) return __uint_as_float(key & 0x7FFFFFFFu);
    if (key >= 0x00800000u) return __uint_as_float(~key);
    return -INFINITY;
}

// Compare-exchange: a keeps the larger value, b the smaller.
__device__ __forceinline__ void ce_desc(float &a, float &b) {
    const float hi = fmaxf(a, b);
    b = fminf(a, b);
    a = hi;
}

// Sorts 16 values descending: the bitonic network (sorted runs of 2, 4, 8, 16, alternately descending
// and ascending until the last merge), 10 stages of 8 compare-exchanges.
__device__ __forceinline__ void sort16_desc(float (&a)[16]) {
#pragma unroll
    for (int size = 2; size <= 16; size <<= 1)
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1)
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int j = i ^ stride;
                if (j > i) {
                    if ((i & size) == 0)
                        ce_desc(a[i], a[j]);
                    else
                        ce_desc(a[j], a[i]);
                }
            }
}

// a <- the 16 largest of a and b, descending (both descending): max(a[i], b[15 - i]) is a bitonic
// sequence holding them, which one bitonic merge (4 stages of 8 compare-exchanges) sorts.
__device__ __forceinline__ void merge_top16_desc(float (&a)[16], const float (&b)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) a[i] = fmaxf(a[i], b[15 - i]);
#pragma unroll
    for (int stride = 8; stride > 0; stride >>= 1)
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int j = i ^ stride;
            if (j > i) ce_desc(a[i], a[j]);
        }
}

__global__ void __launch_bounds__(kSelTcThreads, 1) select_tc_kernel(const __nv_bfloat16 *__restrict__ Q,
                                                           const float *__restrict__ Kbar, int32_t *__restrict__ idx,
                                                           int T_len, int s, int k, int nb, int G) {
    using L = SelTcSmem;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar_mma = reinterpret_cast<uint64_t *>(smem + L::kBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kBar + 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kBar + 16);
    int *cnt_sm = reinterpret_cast<int *>(smem + L::kCnt);          // [2][4][128]
    uint32_t *gt_sm = reinterpret_cast<uint32_t *>(smem + L::kMask);  // [8][128]
    uint32_t *eq_sm = gt_sm + 8 * 128;                                // [8][128]
    float *list_sm = reinterpret_cast<float *>(smem + L::kList);      // [4][128][kSelList]
    float *thr_sm = reinterpret_cast<float *>(smem + L::kThr);        // [128]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.y, t0 = blockIdx.x * kSelTcRows;
    const size_t head_rows = static_cast<size_t>(bh) * T_len;
    const int last = min(t0 + kSelTcRows, T_len) - 1;
    const int nbc = min(last / s, nb);  // blocks scored by some row of the tile (j < b(t))
    const int ngroups = (nbc + 63) / 64;
    const uint32_t sQ = smem_u32(smem + L::kQ), sB = smem_u32(smem + L::kB);

    if (tid == 0) {
        mbar_init(bar_mma, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    // query rows of head (bh * G + hi) -> K-major 128-byte-swizzled tile; rows past T are zero-filled
    auto load_q = [&](int hi) {
        const int u = tid & 15;
        const size_t qrows = (static_cast<size_t>(bh) * G + hi) * T_len;
        for (int row = tid >> 4; row < kSelTcRows; row += kSelTcThreads / 16) {
            const int t = t0 + row;
            const bool valid = t < T_len;
            const uint32_t dst = sQ + (u >> 3) * 16384 + row * 128 + ((((u & 7) ^ (row & 7)) & 7) << 4);
            cp_async_16(dst, Q + (qrows + (valid ? t : 0)) * 128 + u * 8, valid ? 16u : 0u);
        }
        cp_async_wait_all();
        fence_proxy_async_smem();
    };
    if (G == 1) load_q(0);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;
    int phase = 0;  // completed MMA batches (bar_mma phases)
    // Kbar rows 64gi .. 64gi+63 -> hi / mid / lo tiles (K-major, swizzled) of buffer sBb; rows >= nbc are
    // zero.  Lane c4 of a warp takes dims 4c4 .. 4c4+3 of one row: two 128-byte row halves per store.
    // The split of a group of 64 pooled keys: every warp takes 4 rows, one float4 per lane.  The rows are
    // loaded into registers first (load_rows), then split and stored (split_store); the stores are asm with
    // a memory clobber, so a load issued after one would wait for it: one L2 round trip per row.
    constexpr int kRowsPerWarp = 64 / (kSelTcThreads / 32);
    static_assert(64 % (kSelTcThreads / 32) == 0, "64 pooled keys per group over the CTA's warps");
    auto load_rows = [&](int gi, float4 (&vr)[kRowsPerWarp]) {
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) {
            const int j = 64 * gi + warp + i * (kSelTcThreads / 32);
            vr[i] = j < nbc ? __ldg(reinterpret_cast<const float4 *>(Kbar + (static_cast<size_t>(bh) * nb + j) * 128) + lane)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    auto split_store = [&](const float4 (&vr)[kRowsPerWarp], uint32_t sBb) {
        const int c4 = lane;
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) {
            const int jj = warp + i * (kSelTcThreads / 32);
            const float4 v = vr[i];
            const uint32_t h01 = pack_bf16x2(v.x, v.y), h23 = pack_bf16x2(v.z, v.w);
            const float r0 = v.x - __uint_as_float(h01 << 16), r1 = v.y - __uint_as_float(h01 & 0xFFFF0000u);
            const float r2 = v.z - __uint_as_float(h23 << 16), r3 = v.w - __uint_as_float(h23 & 0xFFFF0000u);
            const uint32_t m01 = pack_bf16x2(r0, r1), m23 = pack_bf16x2(r2, r3);
            const uint32_t l01 = pack_bf16x2(r0 - __uint_as_float(m01 << 16), r1 - __uint_as_float(m01 & 0xFFFF0000u));
            const uint32_t l23 = pack_bf16x2(r2 - __uint_as_float(m23 << 16), r3 - __uint_as_float(m23 & 0xFFFF0000u));
            const uint32_t off = (c4 >> 4) * 8192 + jj * 128 + (((((c4 & 15) >> 1) ^ (jj & 7)) & 7) << 4) + (c4 & 1) * 8;
            st_shared_v2(sBb + off, h01, h23);
            st_shared_v2(sBb + 16384 + off, m01, m23);
            st_shared_v2(sBb + 2 * 16384 + off, l01, l23);
        }
        fence_proxy_async_smem();  // generic-proxy tile writes -> tensor-core reads
    };
    // S[:, 64gi ..] (+)= Q [hi | mid | lo]^T, issued by one thread, completion on bar_mma
    auto issue = [&](int gi, uint32_t sBb, bool acc0) {
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int sp = 0; sp < 3; ++sp)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ss(tmem + 64 * gi, smem_desc_sw128(sQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16),
                                smem_desc_sw128(sBb + sp * 16384 + (kk >> 2) * 8192 + (kk & 3) * 32, 16), id,
                                (acc0 || sp > 0 || kk > 0) ? 1u : 0u);
            mma_commit(bar_mma);
        }
    };
    if (G == 1) {
        // the split of group gi is written while the MMAs of group gi-1 run (two buffers: buffer gi & 1
        // was last read by the MMAs of group gi-2, which completed before group gi-1 was issued)
        // the next group's rows are loaded right after this group's split is stored: in flight while the
        // previous group's MMAs complete and this group's are issued
        float4 vr[kRowsPerWarp];
        if (ngroups > 0) load_rows(0, vr);
        for (int gi = 0; gi < ngroups && ok; ++gi) {
            split_store(vr, sB + (gi & 1) * L::kBBuf);
            if (gi + 1 < ngroups) load_rows(gi + 1, vr);
            if (gi > 0) {
                if (!mbar_wait(bar_mma, phase & 1, abort_flag, 0x501)) ok = false;
                ++phase;
            }
            __syncthreads();
            issue(gi, sB + (gi & 1) * L::kBBuf, false);
        }
        if (ok && ngroups > 0) {
            if (!mbar_wait(bar_mma, phase & 1, abort_flag, 0x501)) ok = false;
            ++phase;
        }
    } else {
        for (int gi = 0; gi < ngroups && ok; ++gi) {
            {
                float4 vr[kRowsPerWarp];
                load_rows(gi, vr);
                split_store(vr, sB);
            }
            // with grouped query heads the group's tiles are added one after another into the same scores
            for (int hi = 0; hi < G && ok; ++hi) {
                load_q(hi);  // the previous batch's MMAs have read the tile (waited below)
                __syncthreads();
                issue(gi, sB, hi > 0);
                // the split tiles and the query tile are rewritten only after these MMAs have read them
                if (!mbar_wait(bar_mma, phase & 1, abort_flag, 0x501)) ok = false;
                ++phase;
            }
        }
    }
    // one decision for the whole CTA: the loads below are warp-collective and the row groups meet on
    // named barriers, so every thread must take the same branch
    ok = __syncthreads_and(ok ? 1 : 0) != 0;
    tc_fence_after();

    // ---- top-(k-1) per row: thread <-> row, four warps (column groups) per row group ----
    const int rg = warp & 3, cg = warp >> 2;  // row group, column group
    const int r = rg * 32 + lane;
    const int t = t0 + r;
    const bool valid_row = t < T_len;
    const int bt = t / s;
    const int n = valid_row ? min(bt, nb) : 0;  // candidates j < b(t)  (uniform over a warp: s >= 64)
    const int want = min(k - 1, n);
    const int nch = (nbc + 31) / 32;           // score chunks of the tile (<= 8)
    const uint32_t lane_off = static_cast<uint32_t>(rg * 32) << 16;
    float x[2][32];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int c = cg + 4 * i;
        if (ok && c < nch) {  // warp-uniform
            uint32_t v[32];
            tmem_ld32_async(tmem + lane_off + 32 * c, v);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) x[i][e] = (32 * c + e < n) ? __uint_as_float(v[e]) : __int_as_float(0x7FC00000);
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) x[i][e] = __int_as_float(0x7FC00000);  // NaN: never counted
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 256);

    // chunks of this warp that hold candidates of its rows (n is uniform over the warp)
    const int mych = (cg < (n + 31) / 32 ? 1 : 0) + (cg + 4 < (n + 31) / 32 ? 1 : 0);
    auto count_ge = [&](float f) {
        int c = 0;
        if (mych > 0) {
#pragma unroll
            for (int e = 0; e < 32; ++e) c += (x[0][e] >= f) ? 1 : 0;
        }
        if (mych > 1) {
#pragma unroll
            for (int e = 0; e < 32; ++e) c += (x[1][e] >= f) ? 1 : 0;
        }
        return c;
    };
    const bool search = ok && want > 0 && want < n;  // uniform over the row group
    float ft = 0.f;     // threshold: the want-th largest score of the row
    bool exact = false;  // exactly want scores at or above ft (otherwise: above ft, then ties lowest first)
    if (k - 1 <= kSelList) {
        // Each thread forms the kSelList largest of its candidates in registers (a descending list):
        // groups of 16 sorted by a bitonic network, each merged into the running list by keeping the
        // larger of a[i] and b[15-i] (a bitonic sequence holding the 16 largest) and one bitonic merge
        // (880 min/max per 64 candidates, against 2,048 for passing each candidate down a 16-long
        // compare-exchange chain); thread cg = 0 of each row then merges the four threads' lists in
        // shared memory up to the want-th value.
        float lst[kSelList];
        if (search) {
            float g[kSelList];
            auto take = [&](const float (&src)[32], int half, float (&dst)[kSelList]) {
#pragma unroll
                for (int e = 0; e < kSelList; ++e) {
                    const float v = src[half * kSelList + e];
                    dst[e] = (v == v) ? v : -INFINITY;  // non-candidates (NaN) never enter
                }
                sort16_desc(dst);
            };
            if (mych > 0) {
                take(x[0], 0, lst);
                take(x[0], 1, g);
                merge_top16_desc(lst, g);
            } else {
#pragma unroll
                for (int q = 0; q < kSelList; ++q) lst[q] = -INFINITY;
            }
            if (mych > 1) {
                take(x[1], 0, g);
                merge_top16_desc(lst, g);
                take(x[1], 1, g);
                merge_top16_desc(lst, g);
            }
            float4 *dst = reinterpret_cast<float4 *>(list_sm + (cg * 128 + r) * kSelList);
#pragma unroll
            for (int q = 0; q < kSelList / 4; ++q)
                dst[q] = make_float4(lst[4 * q], lst[4 * q + 1], lst[4 * q + 2], lst[4 * q + 3]);
        }
        if (search) named_barrier(1 + rg, 128);
        if (search && cg == 0) {
            const float *l0 = list_sm + r * kSelList, *l1 = l0 + 128 * kSelList, *l2 = l1 + 128 * kSelList,
                        *l3 = l2 + 128 * kSelList;
            int p0 = 0, p1 = 0, p2 = 0, p3 = 0;
            float h0 = l0[0], h1 = l1[0], h2 = l2[0], h3 = l3[0], t = -INFINITY;
            for (int q = 0; q < want; ++q) {
                const float m01 = fmaxf(h0, h1), m23 = fmaxf(h2, h3);
                t = fmaxf(m01, m23);
                if (h0 == t) {
                    ++p0;
                    h0 = p0 < kSelList ? l0[p0] : -INFINITY;
                } else if (h1 == t) {
                    ++p1;
                    h1 = p1 < kSelList ? l1[p1] : -INFINITY;
                } else if (h2 == t) {
                    ++p2;
                    h2 = p2 < kSelList ? l2[p2] : -INFINITY;
                } else {
                    ++p3;
                    h3 = p3 < kSelList ? l3[p3] : -INFINITY;
                }
            }
            thr_sm[r] = t;
        }
        if (search) named_barrier(1 + rg, 128);
        if (search) ft = thr_sm[r];
    } else {
        // the row group's four warps meet on named barrier 1 + rg (128 threads)
        uint32_t tau = 0u;
        if (search) {
            bool done = false;
            int step = 0;
            for (int b = 31; b >= 0; --b, ++step) {
                const uint32_t cand = tau | (1u << b);
                const int part = count_ge(key_value(cand));
                int *cs = cnt_sm + (step & 1) * 512;
                cs[cg * 128 + r] = part;
                named_barrier(1 + rg, 128);
                const int tot = cs[r] + cs[128 + r] + cs[256 + r] + cs[384 + r];
                if (!done && tot >= want) {
                    tau = cand;
                    if (tot == want) exact = done = true;
                }
                if (__all_sync(0xffffffffu, done)) break;  // the same rows and counts in all four warps
            }
        }
        ft = key_value(tau);
    }
    // chosen columns of this warp's chunks: above ft (at or above when exact), and the ties
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int c = cg + 4 * i;
        if (c < nch) {
            uint32_t gm = 0u, em = 0u;
            if (!search) {  // every candidate (non-candidates are NaN)
#pragma unroll
                for (int e = 0; e < 32; ++e) gm |= (x[i][e] == x[i][e] ? 1u : 0u) << e;
            } else if (exact) {
#pragma unroll
                for (int e = 0; e < 32; ++e) gm |= (x[i][e] >= ft ? 1u : 0u) << e;
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    gm |= (x[i][e] > ft ? 1u : 0u) << e;
                    em |= (x[i][e] == ft ? 1u : 0u) << e;
                }
            }
            gt_sm[c * 128 + r] = gm;
            eq_sm[c * 128 + r] = em;
        }
    }
    __syncthreads();
    if (valid_row && ok) {
        // Each of the row's four threads writes the chosen columns of its own chunks, ascending: a chunk's
        // first position is the count of columns above the threshold in the chunks before it plus the ties
        // taken there (ties go lowest column first until want are chosen).
        int above = 0, ab[2] = {0, 0}, eb[2] = {0, 0};
        for (int c = 0; c < nch; ++c) {
            const int pa = __popc(gt_sm[c * 128 + r]), pe = __popc(eq_sm[c * 128 + r]);
            above += pa;
            if (c < cg) ab[0] += pa, eb[0] += pe;
            if (c < cg + 4) ab[1] += pa, eb[1] += pe;
        }
        const int need = search ? want - above : 0;  // ties to take
        int32_t *out = idx + (head_rows + t) * k;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int c = cg + 4 * i;
            if (c >= nch) continue;
            uint32_t m = gt_sm[c * 128 + r], e = eq_sm[c * 128 + r];
            const int ties_before = min(need, eb[i]);
            for (int take = need - ties_before; take > 0 && e != 0u; --take) {
                m |= e & (~e + 1u);  // lowest equal column
                e &= e - 1u;
            }
            int pos = ab[i] + ties_before;
            while (m != 0u && pos < want) {
                out[pos++] = 32 * c + __ffs(m) - 1;
                m &= m - 1u;
            }
        }
        if (cg == 0) {
            out[want] = bt;
            for (int pos = want + 1; pos < k; ++pos) out[pos] = -1;
        }
    }
}

}  // namespace ssa
