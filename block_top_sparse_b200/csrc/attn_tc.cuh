// attn_tc.cuh -- tcgen05 (5th-generation tensor core) attention kernels for
// head dimension 128, bf16 inputs, fp32 accumulation in tensor memory.
//
//  full_fwd_kernel    full causal attention forward, query-major: one CTA per
//                     128-query tile, loops over the causal key tiles with an
//                     online softmax (paper section 3, full attention).
//  sparse_fwd_kernel  block-major sparse forward: one CTA per (head, key block
//                     j) processes, 128 at a time, the queries whose selection
//                     holds j (gathered by row), and writes a normalised fp16
//                     partial output + log-sum-exp per (query, slot); a merge
//                     kernel combines the k partials of each query.
//  (the backward kernel shared by both streams is in attn_bwd.cuh)
//
// Shared-memory operand tiles are "chunks" of R rows x 64 bf16 (128 B rows,
// 128-byte swizzle), see smem_desc_sw128().  Warps 0..3 (128 threads) own one
// tile row each (a query row, or in the backward epilogue a head-dim row);
// warp 4 issues TMA and MMA.
#pragma once

#include "device.cuh"

namespace ssa {

constexpr int kD = 128;         // head dimension of the tensor-core path
constexpr int kTileQ = 128;     // query rows per tile (MMA M)
constexpr int kChunkBytes = 128 * 128;  // 128 rows x 64 bf16

struct Rows {
    // Row source of a query tile of one key/value head's unit.  G query heads read the key head
    // (grouped-query attention; G = 1 for one query head per key head; G is a power of two).
    //  sparse: gathered from the key block's list of entries (t << 8) | slot; a tile holds
    //          128 / G entries, each for all G heads, entry-major (tile row r: entry r / G,
    //          head r % G), so that tile row r of tile it is partial row it * 128 + r of the block;
    //  full:   contiguous query rows from `first` on, the G heads' tiles one head after another.
    const int32_t *list;  // entries, or nullptr for contiguous rows
    int len;              // sparse: entries in the list; full: query rows per head (T - first)
    int first;            // full: first query position
    int k;
    int gshift;           // log2(G)
    int T;
    size_t qrow0;         // row of the group's first query head in the [B*H*T] query tensors
    __device__ __forceinline__ int per_tile() const { return list ? kTileQ >> gshift : kTileQ; }
    __device__ __forceinline__ int tiles_per_head() const { return (len + kTileQ - 1) / kTileQ; }
    __device__ __forceinline__ int ntiles() const {
        return list ? (len + per_tile() - 1) / per_tile() : (tiles_per_head() << gshift);
    }
};

__host__ __device__ __forceinline__ int log2_pow2(int g) {
    int s = 0;
    while ((1 << s) < g) ++s;
    return s;
}

// Query position t and query-tensor row of tile row r of tile `it`; false past the end.  GQ: the
// kernel was instantiated for grouped heads (G > 1); without it the group arithmetic compiles away.
template <bool GQ>
__device__ __forceinline__ bool tile_row(const Rows &R, int it, int r, int &t, size_t &qrow) {
    const int gs = GQ ? R.gshift : 0;
    if (R.list) {
        const int li = (it * kTileQ + r) >> gs;  // it * (128 / G) + r / G
        if (li >= R.len) return false;
        t = __ldg(R.list + li) >> 8;
        qrow = R.qrow0 + t;
        if (GQ) qrow += static_cast<size_t>(r & ((1 << gs) - 1)) * R.T;
        return true;
    }
    const int tph = R.tiles_per_head();
    const int hi = GQ ? it / tph : 0;
    t = R.first + (it - hi * tph) * kTileQ + r;
    qrow = R.qrow0 + static_cast<size_t>(hi) * R.T + t;
    return t < R.T;
}

// Write 32 fp32 values as bf16 into row r, columns [c0, c0+32) of a swizzled
// multi-chunk tile (chunk = 64 columns, chunk stride `cstride` bytes).
__device__ __forceinline__ void store_row32_bf16(uint32_t tile, uint32_t cstride, int r, int c0, const float (&v)[32]) {
    const uint32_t base = tile + (c0 >> 6) * cstride + r * 128;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const uint32_t unit = ((c0 & 63) >> 3) + g;
        const uint32_t addr = base + (((unit ^ (r & 7)) & 7) << 4);
        st_shared_v4(addr, pack_bf16x2(v[8 * g + 0], v[8 * g + 1]), pack_bf16x2(v[8 * g + 2], v[8 * g + 3]),
                     pack_bf16x2(v[8 * g + 4], v[8 * g + 5]), pack_bf16x2(v[8 * g + 6], v[8 * g + 7]));
    }
}

// ---------------------------------------------------------------------------
// MMA sequences (issued by one thread).
// ---------------------------------------------------------------------------

// D[128 x N] = A[128 x 128] * B[N x 128]^T with A, B K-major over K = 128
// (two 64-wide chunks each; A chunk stride 16 KB, B chunk stride b_cstride).
__device__ __forceinline__ void mma_k128_kmajor(uint32_t d_tmem, uint32_t a, uint32_t b, uint32_t b_cstride,
                                                uint32_t idesc) {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const uint64_t da = smem_desc_sw128(a + (kk >> 2) * kChunkBytes + (kk & 3) * 32, 16);
        const uint64_t db = smem_desc_sw128(b + (kk >> 2) * b_cstride + (kk & 3) * 32, 16);
        mma_bf16_ss(d_tmem, da, db, idesc, kk > 0 ? 1u : 0u);
    }
}

// ---------------------------------------------------------------------------
// Full causal attention forward, two query tiles per CTA in ping-pong.
// grid = B*H*ceil(T/256) (query heads; head h reads key/value head h / G), heaviest
// query blocks first; block = 384 threads.
//   warpgroup x in {0, 1} owns query tile x (rows 256*qb + 128*x + row): online
//   softmax over the key tiles 0..diag(x) with lazy rescaling of O (only when the
//   running maximum grows by more than 2^8), P written as bf16 pairs over S in
//   tensor memory;
//   warp 8 issues S_a(0), S_b(0), then per key tile n:
//     PV_a(n), S_a(n+1), PV_b(n), S_b(n+1)
//   so that one warpgroup's softmax overlaps the other's MMAs;
//   warp 9 streams K/V tiles by TMA through a 2-stage ring; warps 10-11 idle.
// smem: Q_a, Q_b 64 KB | K/V 2 stages x 64 KB | barriers
// tmem: S_a 0, S_b 128, O_a 256, O_b 384 (512 allocated).
// ---------------------------------------------------------------------------
struct FullFwdSmem {
    static constexpr int kQ = 0;                              // [2 tiles] x 32 KB
    static constexpr int kK = kQ + 2 * 2 * kChunkBytes;       // [2 stages] x 32 KB
    static constexpr int kV = kK + 2 * 2 * kChunkBytes;       // [2 stages] x 32 KB
    static constexpr int kBar = kV + 2 * 2 * kChunkBytes;
    static constexpr int kTotal = kBar + 256;
};

// 384 threads launched with 168 registers each (64,512); softmax warpgroups grow
// to 224 and the MMA / producer warpgroup shrinks to 56: 2*128*224 + 128*56 = 64,512.
constexpr int kFullFwdThreads = 384;

__global__ void __launch_bounds__(kFullFwdThreads, 1)
    full_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, __nv_bfloat16 *__restrict__ O,
                    __nv_bfloat16 *__restrict__ O_lo, float *__restrict__ lse, int BH, int T, int G,
                    float scale_log2) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + FullFwdSmem::kBar);
    uint64_t *bar_q = bars + 0;
    uint64_t *bar_kv_full = bars + 1;   // [2]
    uint64_t *bar_kv_empty = bars + 3;  // [2]
    uint64_t *bar_s_full = bars + 5;    // [2 tiles]
    uint64_t *bar_p_full = bars + 7;    // [2 tiles]
    uint64_t *bar_o_full = bars + 9;    // [2 tiles]
    uint64_t *bar_final = bars + 11;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 13);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 14);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nqb = (T + 255) / 256;
    int bh, u;
    unit_order(blockIdx.x, BH, nqb, bh, u);
    const int qb = nqb - 1 - u;  // heaviest query blocks first
    const int row0 = bh * T;              // first tensor-map row of this query head
    const int krow0 = (bh / G) * T;       // first row of its key/value head
    const int q0 = qb * 256;              // first query of tile a; tile b starts at q0 + 128
    // key tiles 0 .. diag: tile a ends at key tile 2qb, tile b at 2qb+1
    const int nkv_a = 2 * qb + 1, nkv_b = 2 * qb + 2;

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_kv_full + i, 1);
            mbar_init(bar_kv_empty + i, 1);
            mbar_init(bar_s_full + i, 1);
            mbar_init(bar_p_full + i, 128);
            mbar_init(bar_o_full + i, 1);
        }
        mbar_init(bar_final, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= 8) regs_shrink<56>();
    if (warp == 9) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            mbar_arrive_expect_tx(bar_q, 4 * kChunkBytes);
            for (int x = 0; x < 2; ++x) {
                uint8_t *q = smem + FullFwdSmem::kQ + x * 2 * kChunkBytes;
                tma_load_2d(&tmQ, bar_q, q, 0, row0 + q0 + 128 * x);
                tma_load_2d(&tmQ, bar_q, q + kChunkBytes, 64, row0 + q0 + 128 * x);
            }
            for (int n = 0; n < nkv_b; ++n) {
                const int st = n & 1;
                if (n >= 2 && !mbar_wait(bar_kv_empty + st, ((n >> 1) - 1) & 1, abort_flag, 0x101)) break;
                mbar_arrive_expect_tx(bar_kv_full + st, 4 * kChunkBytes);
                uint8_t *k = smem + FullFwdSmem::kK + st * 2 * kChunkBytes;
                uint8_t *v = smem + FullFwdSmem::kV + st * 2 * kChunkBytes;
                tma_load_2d(&tmK, bar_kv_full + st, k, 0, krow0 + n * kTileQ);
                tma_load_2d(&tmK, bar_kv_full + st, k + kChunkBytes, 64, krow0 + n * kTileQ);
                tma_load_2d(&tmV, bar_kv_full + st, v, 0, krow0 + n * kTileQ);
                tma_load_2d(&tmV, bar_kv_full + st, v + kChunkBytes, 64, krow0 + n * kTileQ);
            }
        }
    } else if (warp == 8) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idS = idesc_bf16(128, 128, false, false);
            const uint32_t idO = idesc_bf16(128, 128, false, true);
            const uint32_t sQ = smem_u32(smem + FullFwdSmem::kQ);
            const uint32_t sK = smem_u32(smem + FullFwdSmem::kK), sV = smem_u32(smem + FullFwdSmem::kV);
            auto issue_S = [&](int x, int n) {
                mma_k128_kmajor(tmem + 128 * x, sQ + x * 2 * kChunkBytes, sK + (n & 1) * 2 * kChunkBytes, kChunkBytes,
                                idS);
                mma_commit(bar_s_full + x);
            };
            auto issue_PV = [&](int x, int n) {
                // O_x += P_x V_n : A = P from tensor memory (bf16 pairs over S_x), B = V [kv rows x d] MN-major
                const uint32_t vb = sV + (n & 1) * 2 * kChunkBytes;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ts(tmem + 256 + 128 * x, tmem + 128 * x + kk * 8, smem_desc_sw128(vb + kk * 2048, kChunkBytes),
                                idO, (n > 0 || kk > 0) ? 1u : 0u);
                mma_commit(bar_o_full + x);
            };
            bool ok = mbar_wait(bar_q, 0, abort_flag, 0x102) && mbar_wait(bar_kv_full, 0, abort_flag, 0x103);
            if (ok) {
                tc_fence_after();
                issue_S(0, 0);
                issue_S(1, 0);
            }
            for (int n = 0; ok && n < nkv_b; ++n) {
                bool next_ready = false;
                auto wait_next = [&]() {
                    if (!next_ready) {
                        next_ready = true;
                        if (!mbar_wait(bar_kv_full + ((n + 1) & 1), ((n + 1) >> 1) & 1, abort_flag, 0x104)) return false;
                        tc_fence_after();
                    }
                    return true;
                };
                if (n < nkv_a) {
                    if (!mbar_wait(bar_p_full + 0, n & 1, abort_flag, 0x105)) break;
                    tc_fence_after();
                    issue_PV(0, n);
                    if (n + 1 < nkv_a) {
                        if (!wait_next()) break;
                        issue_S(0, n + 1);
                    }
                }
                if (!mbar_wait(bar_p_full + 1, n & 1, abort_flag, 0x106)) break;
                tc_fence_after();
                issue_PV(1, n);
                if (n + 1 < nkv_b) {
                    if (!wait_next()) break;
                    issue_S(1, n + 1);
                }
                mma_commit(bar_kv_empty + (n & 1));  // every MMA reading stage n&1 has been issued
            }
            mma_commit(bar_final);
            mbar_wait(bar_final, 0, abort_flag, 0x107);
        }
    } else if (warp < 8) {
        // ---------------- softmax warpgroup x (thread <-> query row) ----------------
        regs_grow<224>();
        const int x = warp >> 2;
        const int r = ((warp & 3) << 5) | lane;
        const int t = q0 + 128 * x + r;
        const int nkv = x == 0 ? nkv_a : nkv_b;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + 128 * x + lane_off, tO = tmem + 256 + 128 * x + lane_off;
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        for (int n = 0; n < nkv; ++n) {
            if (!mbar_wait(bar_s_full + x, n & 1, abort_flag, 0x108)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sr[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32_async(tS + 32 * c, sr[c]);
            tmem_ld_wait();
            // key n*128 + col is attended when col <= lim (causal on the diagonal tile); masked
            // scores become -inf, on the diagonal tile only
            const int lim = (n == nkv - 1) ? t - n * kTileQ : 127;
            if (n == nkv - 1) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (32 * c + i > lim) sr[c][i] = 0xff800000u;
            }
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int i = 0; i < 32; ++i) mx4[i & 3] = fmaxf(mx4[i & 3], __uint_as_float(sr[c][i]));
            const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * scale_log2;
            float alpha = 1.f;
            if (n == 0) {
                m_used = mx;
            } else if (mx > m_used + 8.f) {
                alpha = fast_exp2(m_used - mx);
                m_used = mx;
            }
            if (n > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                // the previous PV of this tile must be complete before O is rescaled
                if (!mbar_wait(bar_o_full + x, (n - 1) & 1, abort_flag, 0x109)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int c0 = 0; c0 < 128; c0 += 32) {
                    float o[32];
                    tmem_ld32(tO + c0, o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= alpha;
                    tmem_st32(tO + c0, o);
                }
            }
            l *= alpha;
            // probabilities -> P (bf16 pairs) in tensor memory, over the first 64 columns of S
            // (chunk c of S lands in packed columns 16c .. 16c+15; every S value is already in registers)
            // p = 2^(s * scale_log2 - m) in packed pairs
            const uint64_t sl2 = f2_pack(scale_log2, scale_log2), nm = f2_pack(-m_used, -m_used);
            uint64_t l2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t pw[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    float x0, x1;
                    f2_unpack(ffma2(f2_pack(__uint_as_float(sr[c][i]), __uint_as_float(sr[c][i + 1])), sl2, nm), x0,
                              x1);
                    const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
                    l2[(i >> 1) & 1] = fadd2(l2[(i >> 1) & 1], f2_pack(p0, p1));
                    pw[i >> 1] = pack_bf16x2(p0, p1);
                }
                tmem_st16_u(tS + 16 * c, pw);
            }
            {
                float la, lb, lc, ld;
                f2_unpack(l2[0], la, lb);
                f2_unpack(l2[1], lc, ld);
                l += (la + lb) + (lc + ld);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(bar_p_full + x);
        }
        if (ok && mbar_wait(bar_o_full + x, (nkv - 1) & 1, abort_flag, 0x10a)) {
            tc_fence_after();
            const float inv_l = 1.f / l;
            const size_t orow = (static_cast<size_t>(row0) + (t < T ? t : 0)) * kD;
            uint4 *d4 = reinterpret_cast<uint4 *>(O + orow);
            uint4 *l4 = O_lo ? reinterpret_cast<uint4 *>(O_lo + orow) : nullptr;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t orow_v[2][32];
                tmem_ld32_async(tO + 64 * hh, orow_v[0]);  // warp-collective: outside the row branch
                tmem_ld32_async(tO + 64 * hh + 32, orow_v[1]);
                tmem_ld_wait();
                if (t < T) {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const uint32_t *xo = orow_v[q >> 2] + 8 * (q & 3);
                        float v[8];
                        uint32_t hi[4];
#pragma unroll
                        for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(xo[i]) * inv_l;
#pragma unroll
                        for (int i = 0; i < 4; ++i) hi[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
                        d4[8 * hh + q] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                        if (l4) {
                            // the rounding residual o - bf16(o), itself rounded to bf16
                            uint32_t lo[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                lo[i] = pack_bf16x2(v[2 * i] - __uint_as_float(hi[i] << 16),
                                                    v[2 * i + 1] - __uint_as_float(hi[i] & 0xFFFF0000u));
                            l4[8 * hh + q] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                        }
                    }
                }
            }
            if (t < T) lse[static_cast<size_t>(row0) + t] = (m_used + __log2f(l)) * kLn2;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// Sparse forward, block-major, two warpgroups in ping-pong.
// grid = (B*Hkv*nb): CTA i takes unit u = order[i] of the index, key/value head
// bh = u / nb, block j = u % nb (the heaviest units first, the rest head-major so
// that the head's query rows stay in L2); a tile holds 128 / G list
// entries for each of the G query heads reading the key head.  block = 512 threads:
//   warpgroup g (warps 4g .. 4g+3) owns the query tiles it = g, g+2, ... of the
//   block's list: masked softmax over the block's NKV keys, P written back over
//   S in tensor memory as bf16 pairs, then the normalised partial output o / l
//   and the partial log-sum-exp of every (query, slot) at the entry's position
//   in the block's list (each warp stages its 32 rows in shared memory and
//   writes them with two TMA tile stores: a tile's rows are contiguous).  The
//   partial is fp16 (11 significant bits: the merged output, and the D of the
//   backward formed from it, stay far below bf16 rounding) scaled by 2^-e_j,
//   where e_j >= 0 keeps the block's values below 2^15 (e_j = 0 unless some
//   |v| of block j reaches 2^15; stored per block for the merge, with a flag
//   word after the last block that is set when any e_j is not 0);
//   warps 8-11 and 13-15 gather each tile's query rows with cp.async, a
//   half-warp per 256-byte row (a gather's cost is set by the number of warp
//   instructions in flight, so seven warps share it; completion on an mbarrier);
//   warp 12 loads K_j, V_j (TMA) and issues each S(it) as soon as its query
//   rows have landed and each PV(it) as soon as its P is ready (polling both
//   with the non-suspending test_wait, so that a barrier that is not ready
//   cannot hold up the other; S(it) never ahead of PV(it-2), whose P it
//   overwrites), so that one
//   warpgroup's softmax overlaps the other's MMAs and epilogue.
// smem: Q[3] 32 KB each | K, V NKV*256 each | O staging[2] 32 KB each | barriers
// tmem: S/P[2] at 0 / 128, O[2] at 256 / 384 (512 allocated).
// ---------------------------------------------------------------------------
constexpr int kSparseFwdQStages = 3;

template <int NKV>
struct SparseFwdSmem {
    static constexpr int kQ = 0;                          // [kSparseFwdQStages]
    static constexpr int kK = kQ + kSparseFwdQStages * 2 * kChunkBytes;
    static constexpr int kV = kK + 2 * NKV * 128;
    static constexpr int kO = kV + 2 * NKV * 128;         // [2] 2 chunks x 128 rows x 128 B, swizzled
    static constexpr int kOStage = 2 * kChunkBytes;
    static constexpr int kBar = kO + 2 * kOStage;
    static constexpr int kTotal = kBar + 256;
};

// 512 threads launched with 128 registers each; the softmax warpgroups grow to
// 192 and the gather / MMA warpgroups shrink to 64: 2*128*192 + 2*128*64 = 65,536.
constexpr int kSparseFwdThreads = 512;
constexpr int kSparseFwdGatherWarps = 7;

// Gather warp gw (of kSparseFwdGatherWarps) copies the row pairs p = gw, gw + 7, ...
// of a 128-row query tile: half-warp h takes row 2p + h, lane l & 15 its 16-byte
// unit, into the 2-chunk 128-byte-swizzled tile.  Rows past the list are zero-filled.
constexpr int kGatherPairs = (64 + kSparseFwdGatherWarps - 1) / kSparseFwdGatherWarps;

// Query-tensor rows (-1 past the list) of this lane's rows of tile `it`.
template <bool GQ>
__device__ __forceinline__ void gather_rows_load(const Rows &R, int it, int gw, int lane, int (&qrow)[kGatherPairs]) {
#pragma unroll
    for (int q = 0; q < kGatherPairs; ++q) {
        const int p = gw + kSparseFwdGatherWarps * q;
        int t = 0;
        size_t row = 0;
        qrow[q] = (p < 64 && tile_row<GQ>(R, it, 2 * p + (lane >> 4), t, row)) ? static_cast<int>(row) : -1;
    }
}

__device__ __forceinline__ void gather_rows_issue(uint32_t tile, const __nv_bfloat16 *base, int gw, int lane,
                                                  const int (&qrow)[kGatherPairs]) {
    const int u = lane & 15;
#pragma unroll
    for (int q = 0; q < kGatherPairs; ++q) {
        const int p = gw + kSparseFwdGatherWarps * q;
        if (p < 64) {
            const int r = 2 * p + (lane >> 4);
            const uint32_t dst = tile + (u >> 3) * kChunkBytes + r * 128 + ((((u & 7) ^ (r & 7)) & 7) << 4);
            const bool valid = qrow[q] >= 0;
            cp_async_16(dst, base + static_cast<size_t>(valid ? qrow[q] : 0) * kD + u * 8, valid ? 16u : 0u);
        }
    }
}

template <int NKV, bool GQ>
__global__ void __launch_bounds__(kSparseFwdThreads, 1)
    sparse_fwd_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmO, const __nv_bfloat16 *__restrict__ Q,
                      const int32_t *__restrict__ entries, const int32_t *__restrict__ lstart,
                      const int32_t *__restrict__ llen, const int32_t *__restrict__ order,
                      float *__restrict__ lsepart, int32_t *__restrict__ bexp,
                      int BH, int T, int k, int nb, int G, float scale_log2) {
    using L = SparseFwdSmem<NKV>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBar);
    uint64_t *bar_kv = bars + 0;
    uint64_t *bar_s_full = bars + 3;   // [2] tensor-memory buffers
    uint64_t *bar_p_full = bars + 5;   // [2]
    uint64_t *bar_o_full = bars + 7;   // [2]
    uint64_t *bar_final = bars + 11;
    uint64_t *bar_q_full = bars + 16;  // [kSparseFwdQStages] query-row stages landed
    uint64_t *bar_q_free = bars + 20;  // [kSparseFwdQStages] the S MMA reading a stage has completed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 14);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 15);
    uint32_t *vmax_part = reinterpret_cast<uint32_t *>(bars + 24);  // [8] per softmax warp, |v| bits

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int bh, j;  // key/value head, key block, in the index's launch order (heaviest units first)
    {
        const int u = __ldg(order + blockIdx.x);
        bh = u / nb;
        j = u - bh * nb;
    }
    const int kv0 = j * NKV;
    const size_t head_rows = static_cast<size_t>(bh) * T;  // key/value rows of this head
    // this block's list starts at list position obase; its partial-output rows at obase * G
    const size_t obase = static_cast<size_t>(bh) * list_stride(T, k, nb) + lstart[bh * nb + j];
    Rows R;
    R.list = entries + obase;
    R.len = llen[bh * nb + j];
    R.first = 0;
    R.k = k;
    R.gshift = log2_pow2(G);
    R.T = T;
    R.qrow0 = static_cast<size_t>(bh) * G * T;
    const int ntiles = R.ntiles();
    const size_t prow0 = obase * G;  // partial row of tile row 0 of tile 0

    if (threadIdx.x == 0) {
        mbar_init(bar_kv, 1);
        for (int q = 0; q < kSparseFwdQStages; ++q) {
            mbar_init(bar_q_full + q, 32 * kSparseFwdGatherWarps);  // one cp.async arrival per gather lane
            mbar_init(bar_q_free + q, 1);
        }
        for (int g = 0; g < 2; ++g) {
            mbar_init(bar_s_full + g, 1);
            mbar_init(bar_p_full + g, 128);
            mbar_init(bar_o_full + g, 1);
        }
        mbar_init(bar_final, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t sK = smem_u32(smem + L::kK), sV = smem_u32(smem + L::kV);

    if (warp >= 8) regs_shrink<64>();
    if (warp >= 8 && warp != 12) {
        // ---------------- gather warps: query rows of tile it into Q[it & 1] ----------------
        const int gw = warp < 12 ? warp - 8 : warp - 9;
        int tn[kGatherPairs];
        gather_rows_load<GQ>(R, 0, gw, lane, tn);
        for (int it = 0; it < ntiles; ++it) {
            const int qs = it % kSparseFwdQStages;
            // stage qs is free once the S MMA of tile it-3 has completed (one lane waits for the warp);
            // the stage's own barrier completes once per use, so its phases cannot run ahead
            bool ok = true;
            if (lane == 0 && it >= kSparseFwdQStages)
                ok = mbar_wait(bar_q_free + qs, (it / kSparseFwdQStages - 1) & 1, abort_flag, 0x208);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            gather_rows_issue(smem_u32(smem + L::kQ + qs * 2 * kChunkBytes), Q, gw, lane, tn);
            cp_async_mbar_arrive_noinc(bar_q_full + qs);
            if (it + 1 < ntiles) gather_rows_load<GQ>(R, it + 1, gw, lane, tn);  // in flight during the next wait
        }
        cp_async_wait_all();
    } else if (warp == 12) {
        if (lane == 0) {
            mbar_arrive_expect_tx(bar_kv, 4 * NKV * 128);
            tma_load_2d(&tmK, bar_kv, smem + L::kK, 0, static_cast<int>(head_rows) + kv0);
            tma_load_2d(&tmK, bar_kv, smem + L::kK + NKV * 128, 64, static_cast<int>(head_rows) + kv0);
            tma_load_2d(&tmV, bar_kv, smem + L::kV, 0, static_cast<int>(head_rows) + kv0);
            tma_load_2d(&tmV, bar_kv, smem + L::kV + NKV * 128, 64, static_cast<int>(head_rows) + kv0);
            const uint32_t idS = idesc_bf16(128, NKV, false, false);
            const uint32_t idO = idesc_bf16(128, 128, false, true);
            bool ok = mbar_wait(bar_kv, 0, abort_flag, 0x201);
            // S(it) overwrites the P of tile it-2 in the same tensor-memory columns: it is issued
            // only after PV(it-2) (tensor-core operations run in issue order).
            int is = 0, ip = 0;  // next S and next PV to issue
            uint64_t t_idle = globaltimer_ns();
            while (ok && ip < ntiles) {
                bool progressed = false;
                if (ip < is && mbar_test_wait(bar_p_full + (ip & 1), (ip >> 1) & 1)) {
                    const int g = ip & 1;
                    tc_fence_after();
                    // O_g = P_g V : A = P from tensor memory (bf16 pairs over S_g), B = V [NKV x d] MN-major
#pragma unroll
                    for (int kk = 0; kk < NKV / 16; ++kk)
                        mma_bf16_ts(tmem + 256 + 128 * g, tmem + 128 * g + kk * 8,
                                    smem_desc_sw128(sV + kk * 2048, NKV * 128), idO, kk > 0 ? 1u : 0u);
                    mma_commit(bar_o_full + g);
                    ++ip;
                    progressed = true;
                }
                if (is < ntiles && is < ip + 2 &&
                    mbar_test_wait(bar_q_full + is % kSparseFwdQStages, (is / kSparseFwdQStages) & 1)) {
                    const int g = is & 1;
                    fence_proxy_async_smem();  // cp.async-written rows -> tensor-core reads
                    tc_fence_after();
                    mma_k128_kmajor(tmem + 128 * g,
                                    smem_u32(smem + L::kQ + (is % kSparseFwdQStages) * 2 * kChunkBytes), sK,
                                    NKV * 128, idS);
                    mma_commit(bar_s_full + g);
                    mma_commit(bar_q_free + is % kSparseFwdQStages);
                    ++is;
                    progressed = true;
                }
                if (progressed) {
                    t_idle = globaltimer_ns();
                } else if (*abort_flag) {
                    ok = false;
                } else if (globaltimer_ns() - t_idle > kWaitLimitNs) {
                    *abort_flag = 1;
                    record_error(ERR_TIMEOUT, 0x202);
                    ok = false;
                }
            }
            mma_commit(bar_final);
            mbar_wait(bar_final, 0, abort_flag, 0x205);
        }
    } else if (warp < 8) {
        regs_grow<192>();
        const int g = warp >> 2;                  // warpgroup: tiles g, g+2, ...
        const int r = ((warp & 3) << 5) | lane;   // tile row
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t sO = smem_u32(smem + L::kO + g * L::kOStage);  // this warpgroup's staging tile
        const uint32_t tS = tmem + 128 * g + lane_off, tO = tmem + 256 + 128 * g + lane_off;
        // this row's query position (-1 past the list) is loaded one tile ahead
        auto row_t = [&](int it) {
            int t = -1;
            size_t qrow;
            return (it < ntiles && tile_row<GQ>(R, it, r, t, qrow)) ? t : -1;
        };
        int t_n = row_t(g);
        // range exponent of the block: max |v| over V_j (bf16 in shared memory; the layout does
        // not matter for a maximum), reduced over the 256 softmax threads
        int e_blk = 0;
        {
            bool okv = mbar_wait(bar_kv, 0, abort_flag, 0x209);
            uint32_t m = 0u;
            if (okv) {
                constexpr int kBytesPer = 2 * NKV * 128 / 256;  // V_j bytes per softmax thread
                const uint4 *src = reinterpret_cast<const uint4 *>(smem + L::kV + threadIdx.x * kBytesPer);
#pragma unroll
                for (int q = 0; q < kBytesPer / 16; ++q) {
                    const uint4 v = src[q];
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) m = max(m, max((w[i] << 16) & 0x7FFF0000u, w[i] & 0x7FFF0000u));
                }
            }
            m = __reduce_max_sync(0xffffffffu, m);  // |v| as fp32 bits: integer order = value order
            if (lane == 0) vmax_part[warp] = m;
            named_barrier(1, 256);
            uint32_t mm = 0u;
#pragma unroll
            for (int w = 0; w < 8; ++w) mm = max(mm, vmax_part[w]);
            const int ex = static_cast<int>(mm >> 23) - 127;  // floor(log2 max|v|); NaN / inf give 128
            e_blk = min(max(ex - 14, 0), 100);
            if (threadIdx.x == 0) {
                bexp[bh * nb + j] = e_blk;
                if (e_blk > 0) atomicOr(bexp + static_cast<size_t>(BH) * nb, 1);  // some block needs its exponent
            }
        }
        const float escale = __uint_as_float(static_cast<uint32_t>(127 - e_blk) << 23);  // 2^-e
        for (int it = g; it < ntiles; it += 2) {
            const int i = it >> 1;
            const int t_row = t_n;
            if (it + 2 < ntiles) t_n = row_t(it + 2);
            const bool valid = t_row >= 0;
            if (!mbar_wait(bar_s_full + g, i & 1, abort_flag, 0x206)) break;
            tc_fence_after();
            const int lim = valid ? t_row - kv0 : -1;
            uint32_t sr[NKV / 32][32];
#pragma unroll
            for (int c = 0; c < NKV / 32; ++c) tmem_ld32_async(tS + 32 * c, sr[c]);
            tmem_ld_wait();
            // key kv0 + col is attended when col <= lim (causal inside the query's own block);
            // masked scores become -inf, and only warps holding such a row pay for the mask
            if (!__all_sync(0xffffffffu, lim >= NKV - 1)) {
#pragma unroll
                for (int c = 0; c < NKV / 32; ++c)
#pragma unroll
                    for (int i2 = 0; i2 < 32; ++i2)
                        if (32 * c + i2 > lim) sr[c][i2] = 0xff800000u;
            }
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < NKV / 32; ++c)
#pragma unroll
                for (int i2 = 0; i2 < 32; ++i2) mx4[i2 & 3] = fmaxf(mx4[i2 & 3], __uint_as_float(sr[c][i2]));
            const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * scale_log2;
            const float mref = (mx == -INFINITY) ? 0.f : mx;
            // p = 2^(s * scale_log2 - mref) in packed pairs; P (bf16 pairs) goes to tensor memory over
            // the first NKV/2 columns of S
            const uint64_t sl2 = f2_pack(scale_log2, scale_log2), nm = f2_pack(-mref, -mref);
            uint64_t l2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
            for (int c = 0; c < NKV / 32; ++c) {
                uint32_t pw[16];
#pragma unroll
                for (int i2 = 0; i2 < 32; i2 += 2) {
                    float x0, x1;
                    f2_unpack(ffma2(f2_pack(__uint_as_float(sr[c][i2]), __uint_as_float(sr[c][i2 + 1])), sl2, nm), x0,
                              x1);
                    const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
                    l2[(i2 >> 1) & 1] = fadd2(l2[(i2 >> 1) & 1], f2_pack(p0, p1));
                    pw[i2 >> 1] = pack_bf16x2(p0, p1);
                }
                tmem_st16_u(tS + 16 * c, pw);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(bar_p_full + g);
            float la, lb, lc, ld;
            f2_unpack(l2[0], la, lb);
            f2_unpack(l2[1], lc, ld);
            const float l = (la + lb) + (lc + ld);
            const float inv_l = (l > 0.f) ? escale / l : 0.f;
            const size_t orow = prow0 + static_cast<size_t>(it) * kTileQ + r;  // partial row of this tile row
            if (valid) lsepart[orow] = (l > 0.f) ? (mref + __log2f(l)) * kLn2 : -INFINITY;
            // the TMA stores of tile it-2 must have read this warp's staging rows
            if (lane == 0) bulk_wait_read();
            __syncwarp();
            if (!mbar_wait(bar_o_full + g, i & 1, abort_flag, 0x207)) break;
            tc_fence_after();
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t ov[2][32];
                tmem_ld32_async(tO + 64 * hh, ov[0]);
                tmem_ld32_async(tO + 64 * hh + 32, ov[1]);
                tmem_ld_wait();
                // row r of column chunk hh, 128-byte swizzle (conflict-free 16-byte stores)
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint32_t *xo = ov[u >> 2] + 8 * (u & 3);
                    st_shared_v4(sO + hh * kChunkBytes + r * 128 + (((u ^ (r & 7)) & 7) << 4),
                                 pack_half2(__uint_as_float(xo[0]) * inv_l, __uint_as_float(xo[1]) * inv_l),
                                 pack_half2(__uint_as_float(xo[2]) * inv_l, __uint_as_float(xo[3]) * inv_l),
                                 pack_half2(__uint_as_float(xo[4]) * inv_l, __uint_as_float(xo[5]) * inv_l),
                                 pack_half2(__uint_as_float(xo[6]) * inv_l, __uint_as_float(xo[7]) * inv_l));
                }
            }
            fence_proxy_async_smem();  // generic-proxy staging writes -> TMA reads
            __syncwarp();
            if (lane == 0) {
                // rows 32w .. 32w+31 of the tile: the padded list region keeps them inside this block's rows
                const int row0 = static_cast<int>(prow0 + static_cast<size_t>(it) * kTileQ + (r - lane));
                tma_store_2d(&tmO, sO + (r - lane) * 128, 0, row0);
                tma_store_2d(&tmO, sO + kChunkBytes + (r - lane) * 128, 64, row0);
                bulk_commit();
            }
        }
        if (lane == 0) bulk_wait();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace ssa
