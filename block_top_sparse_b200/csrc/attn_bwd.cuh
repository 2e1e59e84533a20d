// attn_bwd.cuh -- tcgen05 attention backward shared by the full and the sparse
// stream (head dimension 128, bf16 inputs, fp32 accumulation).
//
// Key-block-outer: one CTA per key tile (full: 128 keys; the query tiles from
// the diagonal on) or per key block j (sparse: s keys; the 128-row tiles of the
// queries whose selection holds j, gathered by row), of one key/value head: with
// grouped query heads the tiles of all G heads reading it (full: head after
// head; sparse: 128 / G list entries per tile, each for the G heads).  K_j, V_j stay in shared
// memory and the transposed accumulators dV_j^T, dK_j^T stay in tensor memory
// for the whole unit.  Per query tile:
//   S = Q K^T, dP = dO V^T                      (M = 128 query rows)
//   P = exp(scale S - lse)                       -> shared memory, bf16; then
//   dV^T += dO^T P  while  dS = P o (dP - D)     -> shared memory, bf16
//   dK^T += Q^T dS                               (M = head dim 128)
//   dQ = dS K, * scale                           -> added into an fp32 accumulator
// Paper: section 4.2 (keys outside S(t) get no gradient; the selection is a
// constant), FlashAttention-2 style recomputation of P from the saved lse.
//
// Warp roles (640 threads, five warpgroups; registers rebalanced with setmaxnreg):
//   warps 0-7    two warpgroups; warp w owns query row (w & 3)*32 + lane and
//                column half (w >> 2) of the row-wise phase (P, dS), then the
//                dV, dK epilogue;
//   warps 8-11   dQ flush: thread <-> query row; the whole dQ tile leaves tensor
//                memory at once, so the next tile's S can start.  Full stream (a
//                tile's rows are contiguous): columns 0-63 into a 32 KB staging
//                buffer of its own, 64-127 into the P region (free once dQ is
//                computed), added by four TMA tensor reduce-adds issued by one
//                thread.  Sparse stream (gathered rows): each warp adds its 32 rows
//                with coalesced fp32 vector reductions through its own region of
//                the staging buffer;
//   warp 12      MMA issuer (one thread);
//   warp 13      TMA producer (K_j, V_j; contiguous Q / dO tiles of the full stream);
//   warps 14-19  sparse stream: gather the next tile's dO rows once the dV MMAs
//                of the current tile have read dO, then its Q rows once the dK
//                MMAs have read Q, with cp.async (a half-warp per 256-byte row).
//
// Shared memory: Q 32 KB | dO 32 KB | K, V NKV*256 B each | P, dS (NKV/64)*16 KB each |
//                dQ staging 32 KB
// Tensor memory: S / dQ at column 0, dP at 128, dV^T at 256, dK^T at 384 (512).
#pragma once

#include "attn_tc.cuh"

namespace ssa {

template <int NKV>
struct BwdSmem {
    static constexpr int kQ = 0;
    static constexpr int kdO = kQ + 2 * kChunkBytes;
    static constexpr int kK = kdO + 2 * kChunkBytes;
    static constexpr int kV = kK + 2 * NKV * 128;
    static constexpr int kP = kV + 2 * NKV * 128;
    static constexpr int kdS = kP + (NKV / 64) * kChunkBytes;
    static constexpr int kF = kdS + (NKV / 64) * kChunkBytes;  // dQ staging: 128 rows x 256 B
    static constexpr int kBar = kF + 2 * kChunkBytes;
    static constexpr int kTotal = kBar + 256;
};

struct BwdArgs {
    const __nv_bfloat16 *Q, *dO;
    const float *lse, *Dvec;
    float *dQacc;  // sparse stream: fp32 dQ accumulator [B*H*T, 128] (the full stream adds through tmdQ)
    void *dK, *dV;  // bf16, or fp32 when grad_fp32
    const int32_t *entries, *lstart, *llen;  // sparse only
    const int32_t *order;                    // sparse: launch order of the (head, block) units
    int BH, T, k, nb, sparse, accumulate, grad_fp32;
    int G;  // query heads per key/value head; BH counts key/value heads
    float scale, scale_log2;
};

// Four consecutive gradient values of one key row of dV and dK (fp32 in registers) to the
// caller's dV, dK at element offset `off`: bf16 or fp32, added to the existing values in fp32
// first when accumulating (one rounding).
__device__ __forceinline__ void write_grad4(const BwdArgs &a, size_t off, float4 v4, float4 k4) {
    if (a.grad_fp32) {
        float4 *dv4 = reinterpret_cast<float4 *>(static_cast<float *>(a.dV) + off);
        float4 *dk4 = reinterpret_cast<float4 *>(static_cast<float *>(a.dK) + off);
        if (a.accumulate) {
            const float4 ov = *dv4, ok4 = *dk4;
            v4.x += ov.x;
            v4.y += ov.y;
            v4.z += ov.z;
            v4.w += ov.w;
            k4.x += ok4.x;
            k4.y += ok4.y;
            k4.z += ok4.z;
            k4.w += ok4.w;
        }
        *dv4 = v4;
        *dk4 = k4;
        return;
    }
    uint2 *dv2 = reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(a.dV) + off);
    uint2 *dk2 = reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(a.dK) + off);
    if (a.accumulate) {
        const uint2 ov = *dv2, ok2 = *dk2;
        v4.x += __uint_as_float(ov.x << 16);
        v4.y += __uint_as_float(ov.x & 0xFFFF0000u);
        v4.z += __uint_as_float(ov.y << 16);
        v4.w += __uint_as_float(ov.y & 0xFFFF0000u);
        k4.x += __uint_as_float(ok2.x << 16);
        k4.y += __uint_as_float(ok2.x & 0xFFFF0000u);
        k4.z += __uint_as_float(ok2.y << 16);
        k4.w += __uint_as_float(ok2.y & 0xFFFF0000u);
    }
    *dv2 = make_uint2(pack_bf16x2(v4.x, v4.y), pack_bf16x2(v4.z, v4.w));
    *dk2 = make_uint2(pack_bf16x2(k4.x, k4.y), pack_bf16x2(k4.z, k4.w));
}

// 640 threads launched with 96 registers each (61,440); setmaxnreg moves them to
// softmax 2 x 144, flush 96, MMA / producer / gather 2 x 48: 128 * 480 = 61,440.
constexpr int kBwdThreads = 640;
constexpr int kBwdGatherWarps = 6;
constexpr int kBwdGatherPairs = (64 + kBwdGatherWarps - 1) / kBwdGatherWarps;

template <int NKV, bool GQ>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                    const __grid_constant__ CUtensorMap tmdQ, const BwdArgs a) {
    using L = BwdSmem<NKV>;
    constexpr int HALF = NKV / 2;  // S / dP columns per warpgroup
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBar);
    uint64_t *bar_kv = bars + 0, *bar_qdo_full = bars + 1, *bar_sdp_full = bars + 2, *bar_pds_full = bars + 3;
    uint64_t *bar_qdo_free = bars + 4, *bar_dq_full = bars + 5, *bar_dq_empty = bars + 6, *bar_final = bars + 7;
    uint64_t *bar_f_staged = bars + 8, *bar_f_free = bars + 9;  // dQ staging buffer handshakes
    uint64_t *bar_p_free = bars + 12;  // the P region's dQ half has been read by the flush
    uint64_t *bar_epi = bars + 13;     // the dV / dK staging of the epilogue is complete
    // dO has its own load / release barriers (released after the dV MMAs, before Q, which the dK
    // MMAs still read), so that the next tile's dO arrives and its dP runs during dK / dQ
    uint64_t *bar_do_full = bars + 14, *bar_do_free = bars + 15;
    uint64_t *bar_ds_full = bars + 16;  // dS stored (bar_pds_full: P stored)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 10);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 11);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T;
    // Unit order: sparse, the index's (heaviest units first, then head-major); full, head-major
    // with each head's longest unit first.  Head-major keeps the query rows and the dQ
    // accumulator of the head being worked on in L2.
    int bh, kb;  // key/value head, key tile (block)
    if (a.order) {
        const int u = __ldg(a.order + blockIdx.x);
        bh = u / a.nb;
        kb = u - bh * a.nb;
    } else {
        unit_order(blockIdx.x, a.BH, (a.T + NKV - 1) / NKV, bh, kb);
    }
    const int kv0 = kb * NKV;
    const size_t head_rows = static_cast<size_t>(bh) * T;  // key/value rows of this head
    const bool sparse = a.sparse != 0;
    Rows R;
    if (sparse) {
        R.list = a.entries + static_cast<size_t>(bh) * list_stride(T, a.k, a.nb) + a.lstart[bh * a.nb + kb];
        R.len = a.llen[bh * a.nb + kb];
        R.first = 0;
    } else {
        R.list = nullptr;
        R.first = kv0;  // causal: query tiles from the key tile onward, for each of the G heads
        R.len = T - kv0;
    }
    R.k = a.k;
    R.gshift = log2_pow2(a.G);
    R.T = T;
    R.qrow0 = static_cast<size_t>(bh) * a.G * T;
    const int ntiles = R.ntiles();
    // query-tensor row of tile row 0 of contiguous tile it (full stream)
    auto tile_row0 = [&](int it) {
        int t;
        size_t qrow;
        tile_row<GQ>(R, it, 0, t, qrow);
        return static_cast<int>(qrow);
    };

    const uint32_t sQ = smem_u32(smem + L::kQ), sdO = smem_u32(smem + L::kdO), sK = smem_u32(smem + L::kK),
                   sV = smem_u32(smem + L::kV), sP = smem_u32(smem + L::kP), sdS = smem_u32(smem + L::kdS),
                   sF = smem_u32(smem + L::kF);

    if (threadIdx.x == 0) {
        mbar_init(bar_kv, 1);
        mbar_init(bar_qdo_full, sparse ? 32 * kBwdGatherWarps : 1);
        mbar_init(bar_sdp_full, 1);
        mbar_init(bar_pds_full, 256);
        mbar_init(bar_ds_full, 256);
        mbar_init(bar_qdo_free, 1);
        mbar_init(bar_do_full, sparse ? 32 * kBwdGatherWarps : 1);
        mbar_init(bar_do_free, 1);
        mbar_init(bar_dq_full, 1);
        mbar_init(bar_dq_empty, 128);
        mbar_init(bar_final, 1);
        mbar_init(bar_f_staged, 128);
        // full stream: staging buffers released by the thread that issued the TMA reduce-adds
        // once they have read shared memory (P region and staging buffer)
        mbar_init(bar_f_free, 1);
        mbar_init(bar_p_free, 1);
        mbar_init(bar_epi, 256);
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
    const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 384, tdQ = tmem;

    if (warp >= 12) {
        regs_shrink<48>();
        if (warp >= 14) {
            // ---------------- gather warps (sparse stream): Q and dO rows of each tile ----------------
            if (sparse) {
                const int gw = warp - 14, u = lane & 15;
                int tn[kBwdGatherPairs];
                auto load_rows = [&](int it) {  // query-tensor rows, -1 past the list
#pragma unroll
                    for (int q = 0; q < kBwdGatherPairs; ++q) {
                        const int p = gw + kBwdGatherWarps * q;
                        int t = 0;
                        size_t row = 0;
                        tn[q] = (p < 64 && tile_row<GQ>(R, it, 2 * p + (lane >> 4), t, row)) ? static_cast<int>(row) : -1;
                    }
                };
                // this lane's rows of one 256-byte-row tensor into a 2-chunk swizzled tile
                auto gather = [&](uint32_t tile, const __nv_bfloat16 *src) {
#pragma unroll
                    for (int q = 0; q < kBwdGatherPairs; ++q) {
                        const int p = gw + kBwdGatherWarps * q;
                        if (p < 64) {
                            const int r = 2 * p + (lane >> 4);
                            const uint32_t off = (u >> 3) * kChunkBytes + r * 128 + ((((u & 7) ^ (r & 7)) & 7) << 4);
                            const bool valid = tn[q] >= 0;
                            cp_async_16_row(tile + off, src + u * 8, valid ? static_cast<uint32_t>(tn[q]) : 0u,
                                            valid ? 16u : 0u);
                        }
                    }
                };
                load_rows(0);
                bool ok = true;
                for (int it = 0; ok && it < ntiles; ++it) {
                    // dO is free once the dV MMAs of the previous tile have completed, Q once its dK MMAs
                    // have: dO comes first, so that dP of this tile can run while dK, dQ of the previous
                    // one do.  (One wait site for both: the loop runs twice per tile.)
#pragma unroll 1
                    for (int ph = 0; ph < 2; ++ph) {
                        if (lane == 0 && it > 0)
                            ok = mbar_wait(ph == 0 ? bar_do_free : bar_qdo_free, (it - 1) & 1, abort_flag, 0x312 + ph);
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        if (!ok) break;
                        gather(ph == 0 ? sdO : sQ, ph == 0 ? a.dO : a.Q);
                        cp_async_mbar_arrive_noinc(ph == 0 ? bar_do_full : bar_qdo_full);
                    }
                    if (ok && it + 1 < ntiles) load_rows(it + 1);  // in flight during the next wait
                }
                cp_async_wait_all();
            }
        } else if (warp == 13) {
            // ---------------- TMA producer ----------------
            if (lane == 0) {
                const int krow = static_cast<int>(head_rows) + kv0;
                mbar_arrive_expect_tx(bar_kv, 4 * NKV * 128);
                tma_load_2d(&tmK, bar_kv, smem + L::kK, 0, krow);
                tma_load_2d(&tmK, bar_kv, smem + L::kK + NKV * 128, 64, krow);
                tma_load_2d(&tmV, bar_kv, smem + L::kV, 0, krow);
                tma_load_2d(&tmV, bar_kv, smem + L::kV + NKV * 128, 64, krow);
                if (!sparse) {
                    int do_issued = 0, q_issued = 0;
                    for (int it = 0; it < ntiles; ++it) {
                        const int qrow = tile_row0(it);
                        // dO of tile it once the dV MMAs of tile it-1 have read dO
                        if (it > 0 && !mbar_wait(bar_do_free, (it - 1) & 1, abort_flag, 0x314)) break;
                        mbar_arrive_expect_tx(bar_do_full, 2 * kChunkBytes);
                        tma_load_2d(&tmdO, bar_do_full, smem + L::kdO, 0, qrow);
                        tma_load_2d(&tmdO, bar_do_full, smem + L::kdO + kChunkBytes, 64, qrow);
                        do_issued = it + 1;
                        // Q of tile it once the dK MMAs of tile it-1 have read Q
                        if (it > 0 && !mbar_wait(bar_qdo_free, (it - 1) & 1, abort_flag, 0x311)) break;
                        mbar_arrive_expect_tx(bar_qdo_full, 2 * kChunkBytes);
                        tma_load_2d(&tmQ, bar_qdo_full, smem + L::kQ, 0, qrow);
                        tma_load_2d(&tmQ, bar_qdo_full, smem + L::kQ + kChunkBytes, 64, qrow);
                        q_issued = it + 1;
                    }
                    // on an abort, let loads still in flight land before the CTA exits
                    if (do_issued > 0) mbar_drain(bar_do_full, (do_issued - 1) & 1);
                    if (q_issued > 0) mbar_drain(bar_qdo_full, (q_issued - 1) & 1);
                }
            }
        } else if (warp == 12) {
            // ---------------- MMA issuer ----------------
            if (lane == 0) {
                const uint32_t idS = idesc_bf16(128, NKV, false, false);  // S, dP
                const uint32_t idT = idesc_bf16(128, NKV, true, true);    // dV^T, dK^T
                const uint32_t idQ = idesc_bf16(128, 128, false, true);   // dQ
                bool ok = mbar_wait(bar_kv, 0, abort_flag, 0x301);
                for (int it = 0; ok && it < ntiles; ++it) {
                    // dP first (its columns are free once the previous tile's P/dS were formed), then S,
                    // which overwrites the previous tile's dQ once the flush has taken it out
                    if (!mbar_wait(bar_do_full, it & 1, abort_flag, 0x302)) break;
                    if (sparse) fence_proxy_async_smem();  // cp.async-written rows -> tensor-core reads
                    tc_fence_after();
                    mma_k128_kmajor(tdP, sdO, sV, NKV * 128, idS);
                    if (!mbar_wait(bar_qdo_full, it & 1, abort_flag, 0x315)) break;
                    if (sparse) fence_proxy_async_smem();
                    if (it > 0 && !mbar_wait(bar_dq_empty, (it - 1) & 1, abort_flag, 0x303)) break;
                    tc_fence_after();
                    mma_k128_kmajor(tS, sQ, sK, NKV * 128, idS);
                    mma_commit(bar_sdp_full);
                    // dV^T[d x kv] += dO^T P as soon as P is stored (while dS is formed); then
                    // dK^T[d x kv] += Q^T dS   (K = 128 query rows)
                    if (!mbar_wait(bar_pds_full, it & 1, abort_flag, 0x304)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        mma_bf16_ss(tdV, smem_desc_sw128(sdO + kk * 2048, kChunkBytes),
                                    smem_desc_sw128(sP + kk * 2048, kChunkBytes), idT, (it > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(bar_do_free);
                    if (!mbar_wait(bar_ds_full, it & 1, abort_flag, 0x316)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        mma_bf16_ss(tdK, smem_desc_sw128(sQ + kk * 2048, kChunkBytes),
                                    smem_desc_sw128(sdS + kk * 2048, kChunkBytes), idT, (it > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(bar_qdo_free);
                    // dQ[q x d] = dS K   (K = NKV keys)
#pragma unroll
                    for (int kk = 0; kk < NKV / 16; ++kk) {
                        mma_bf16_ss(tdQ, smem_desc_sw128(sdS + (kk >> 2) * kChunkBytes + (kk & 3) * 32, 16),
                                    smem_desc_sw128(sK + kk * 2048, NKV * 128), idQ, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(bar_dq_full);
                }
                mma_commit(bar_final);
                mbar_wait(bar_final, 0, abort_flag, 0x305);
            }
        }
    } else if (warp >= 8) {
        // ---------------- dQ flush (thread <-> query row of the tile) ----------------
        // (stays at the 96 registers it was launched with)
        const int r = ((warp & 3) << 5) | lane;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        if (!sparse) {
            for (int it = 0; it < ntiles; ++it) {
                if (!mbar_wait(bar_dq_full, it & 1, abort_flag, 0x307)) break;
                tc_fence_after();
                // both staging buffers' previous contents (tile it-1) have been read by the TMA unit
                if (it > 0 && !mbar_wait(bar_f_free, (it - 1) & 1, abort_flag, 0x30b)) break;
                // Full stream: columns 32c .. 32c+31 as a 128-row x 128-byte swizzled chunk (chunks
                // 0, 1 in sF, 2, 3 in the P region), added by four TMA tensor reduce-adds
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                    uint32_t g[2][32];
                    tmem_ld32_async(tdQ + lane_off + 64 * c2, g[0]);
                    tmem_ld32_async(tdQ + lane_off + 64 * c2 + 32, g[1]);
                    tmem_ld_wait();
                    if (c2 == 1) {
                        tc_fence_before();
                        mbar_arrive(bar_dq_empty);  // dQ has left tensor memory: the next S may overwrite it
                    }
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const uint32_t base = (c2 == 0 ? sF : sP) + cc * kChunkBytes + r * 128;
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const uint32_t *x = g[cc] + 4 * q;
                            st_shared_v4(base + (((q ^ r) & 7) << 4), __float_as_uint(__uint_as_float(x[0]) * a.scale),
                                         __float_as_uint(__uint_as_float(x[1]) * a.scale),
                                         __float_as_uint(__uint_as_float(x[2]) * a.scale),
                                         __float_as_uint(__uint_as_float(x[3]) * a.scale));
                        }
                    }
                }
                fence_proxy_async_smem();  // generic-proxy staging writes -> TMA reads
                mbar_arrive(bar_f_staged);
                if (r == 0) {
                    if (!mbar_wait(bar_f_staged, it & 1, abort_flag, 0x30a)) break;
                    // rows past T in the last tile hold exact zeros (P = 0 there); rows past the
                    // tensor are clipped by the TMA unit
                    const int row0 = tile_row0(it);
                    // the P-region chunks first, in a group of their own, so that P is released early
                    tma_reduce_add_2d(&tmdQ, sP, 64, row0);
                    tma_reduce_add_2d(&tmdQ, sP + kChunkBytes, 96, row0);
                    bulk_commit();
                    tma_reduce_add_2d(&tmdQ, sF, 0, row0);
                    tma_reduce_add_2d(&tmdQ, sF + kChunkBytes, 32, row0);
                    bulk_commit();
                    bulk_wait_read_all_but_1();
                    mbar_arrive(bar_p_free);
                    bulk_wait_read();
                    mbar_arrive(bar_f_free);
                }
            }
            if (r == 0) bulk_wait();  // the TMA reduce-adds have completed
        } else {
            // Sparse stream (gathered rows): each warp adds its 32 rows of the tile's dQ (scaled,
            // fp32) into the fp32 accumulator rows of their queries with vector reductions.  One
            // 64-column half at a time goes through the warp's own 8 KB region of the staging buffer
            // (row rl: 16-byte unit q at position q ^ (rl & 15), conflict-free for the row-owner
            // writes and for the reads below), then each half-warp adds one 256-byte row half per
            // instruction.  Columns 64-127 wait in registers, so the whole tile leaves tensor
            // memory at once.  No cross-warp barrier: a warp only reuses its own region.
            const uint32_t stg = sF + static_cast<uint32_t>(warp & 3) * 8192u;
            auto stage = [&](const uint32_t (&g)[32], int q0) {
#pragma unroll
                for (int q8 = 0; q8 < 8; ++q8) {
                    const int q = q0 + q8;
                    const uint32_t *x = g + 4 * q8;
                    st_shared_v4(stg + lane * 256 + (((q ^ lane) & 15) << 4),
                                 __float_as_uint(__uint_as_float(x[0]) * a.scale),
                                 __float_as_uint(__uint_as_float(x[1]) * a.scale),
                                 __float_as_uint(__uint_as_float(x[2]) * a.scale),
                                 __float_as_uint(__uint_as_float(x[3]) * a.scale));
                }
            };
            auto add_half = [&](int hf, int t_mine) {
                __syncwarp();
                const int u = lane & 15;
#pragma unroll 4
                for (int i = 0; i < 16; ++i) {
                    const int rl = 2 * i + (lane >> 4);
                    const int t_dst = __shfl_sync(0xffffffffu, t_mine, rl);  // query-tensor row
                    float4 v;
                    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                                 : "r"(stg + rl * 256 + (((u ^ rl) & 15) << 4)));
                    if (t_dst >= 0)
                        atomicAdd(reinterpret_cast<float4 *>(a.dQacc + static_cast<size_t>(t_dst) * kD + 64 * hf) + u, v);
                }
                __syncwarp();
            };
            // row r's query-tensor row (-1 past the list), loaded one tile ahead
            auto row_of = [&](int it) {
                int t;
                size_t qrow;
                return (it < ntiles && tile_row<GQ>(R, it, r, t, qrow)) ? static_cast<int>(qrow) : -1;
            };
            int q_n = row_of(0);
            for (int it = 0; it < ntiles; ++it) {
                const int t_mine = q_n;  // destination row of this thread's dQ row
                q_n = row_of(it + 1);
                if (!mbar_wait(bar_dq_full, it & 1, abort_flag, 0x307)) break;
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t g[32];
                    tmem_ld32_async(tdQ + lane_off + 32 * c, g);
                    tmem_ld_wait();
                    stage(g, 8 * c);
                }
                uint32_t hi[2][32];
                tmem_ld32_async(tdQ + lane_off + 64, hi[0]);
                tmem_ld32_async(tdQ + lane_off + 96, hi[1]);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(bar_dq_empty);  // dQ has left tensor memory: the next S may overwrite it
                add_half(0, t_mine);
                stage(hi[0], 0);
                stage(hi[1], 8);
                add_half(1, t_mine);
            }
        }
    } else {
        // ---------------- softmax / dS warpgroups ----------------
        regs_grow<144>();
        const int r = ((warp & 3) << 5) | lane;  // tile row
        const int h = warp >> 2;                 // column half
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        bool ok = true;
        // Row data is fetched ahead: the query position of tile it+2 and the lse, D of tile it+1
        // are loaded while tile it is processed (the sparse stream's lse / D addresses depend on
        // the position loaded from the list), so no dependent global load sits between two tiles.
        int t_n1 = 0, t_n2 = 0;
        size_t q_n1 = 0, q_n2 = 0;
        bool v_n1 = ntiles > 0 && tile_row<GQ>(R, 0, r, t_n1, q_n1);
        float lse_n = v_n1 ? __ldg(a.lse + q_n1) : 0.f;
        float D_n = v_n1 ? __ldg(a.Dvec + q_n1) : 0.f;
        bool v_n2 = ntiles > 1 && tile_row<GQ>(R, 1, r, t_n2, q_n2);
        for (int it = 0; it < ntiles; ++it) {
            const bool valid = v_n1;
            const int t = t_n1;
            const float lse2 = lse_n * kLog2e;
            const float Dt = D_n;
            v_n1 = v_n2;
            t_n1 = t_n2;
            q_n1 = q_n2;
            lse_n = v_n1 ? __ldg(a.lse + q_n1) : 0.f;
            D_n = v_n1 ? __ldg(a.Dvec + q_n1) : 0.f;
            v_n2 = it + 2 < ntiles && tile_row<GQ>(R, it + 2, r, t_n2, q_n2);
            if (!mbar_wait(bar_sdp_full, it & 1, abort_flag, 0x306)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // key kv0 + col is attended when col <= lim (causal inside the diagonal block)
            const int lim = valid ? t - kv0 - h * HALF : -1;
            const uint64_t sl2 = f2_pack(a.scale_log2, a.scale_log2), nl2 = f2_pack(-lse2, -lse2),
                           nD = f2_pack(-Dt, -Dt);
            // P = 2^(s * scale_log2 - lse2) first, stored so that the dV MMAs start while dS is formed
            float p[HALF];
#pragma unroll
            for (int c = 0; c < HALF / 32; ++c) {
                uint32_t sraw[32];
                tmem_ld32_async(tS + lane_off + h * HALF + 32 * c, sraw);
                tmem_ld_wait();
                // masked scores become -inf (only warps holding a masked column pay for it)
                if (!__all_sync(0xffffffffu, lim >= 32 * c + 31)) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (32 * c + i > lim) sraw[i] = 0xff800000u;
                }
                float sv[32];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    float x0, x1;
                    f2_unpack(ffma2(f2_pack(__uint_as_float(sraw[i]), __uint_as_float(sraw[i + 1])), sl2, nl2), x0, x1);
                    sv[i] = fast_exp2(x0);
                    sv[i + 1] = fast_exp2(x1);
                    p[32 * c + i] = sv[i];
                    p[32 * c + i + 1] = sv[i + 1];
                }
                // full stream: the previous tile's dQ staged over P (and dS for 64-key units) has been read
                if (!sparse && c == 0 && it > 0) ok = mbar_wait(bar_p_free, (it - 1) & 1, abort_flag, 0x30d);
                store_row32_bf16(sP, kChunkBytes, r, h * HALF + 32 * c, sv);
            }
            if (!ok) break;
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bar_pds_full);
            // dS = P o (dP - D), in packed pairs
#pragma unroll
            for (int c = 0; c < HALF / 32; ++c) {
                uint32_t draw[32];
                tmem_ld32_async(tdP + lane_off + h * HALF + 32 * c, draw);
                tmem_ld_wait();
                float dp[32];
#pragma unroll
                for (int i = 0; i < 32; i += 2)
                    f2_unpack(fmul2(f2_pack(p[32 * c + i], p[32 * c + i + 1]),
                                    fadd2(f2_pack(__uint_as_float(draw[i]), __uint_as_float(draw[i + 1])), nD)),
                              dp[i], dp[i + 1]);
                store_row32_bf16(sdS, kChunkBytes, r, h * HALF + 32 * c, dp);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bar_ds_full);
        }
        // Epilogue.  dV^T / dK^T (thread <-> head-dim row r, key columns of its half) are restaged in
        // fp32 as [key][dim] rows over the idle operand buffers (dV over Q/dO, dK over K/V, NKV rows of
        // 512 bytes each), then every warp writes whole 256-byte bf16 rows with 16-byte accesses, adding
        // the existing gradient in fp32 first when asked (one rounding).
        if (ok && !mbar_wait(bar_final, 0, abort_flag, 0x30c)) ok = false;
        tc_fence_after();
        const uint32_t sdv = sQ, sdk = sK;
        if (ok) {
#pragma unroll
            for (int c0 = h * HALF; c0 < (h + 1) * HALF; c0 += 32) {
                uint32_t rv[32], rk[32];
                tmem_ld32_async(tdV + lane_off + c0, rv);
                tmem_ld32_async(tdK + lane_off + c0, rk);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float vv = ntiles > 0 ? __uint_as_float(rv[i]) : 0.f;
                    const float kq = ntiles > 0 ? __uint_as_float(rk[i]) * a.scale : 0.f;
                    // a warp stores 32 consecutive dims of one key row: 128 contiguous bytes
                    asm volatile("st.shared.f32 [%0], %1;" ::"r"(sdv + (c0 + i) * 512 + r * 4), "f"(vv) : "memory");
                    asm volatile("st.shared.f32 [%0], %1;" ::"r"(sdk + (c0 + i) * 512 + r * 4), "f"(kq) : "memory");
                }
            }
        }
        mbar_arrive(bar_epi);
        if (ok && !mbar_wait(bar_epi, 0, abort_flag, 0x30e)) ok = false;
        if (ok) {
            // warp w writes key rows w, w+8, ...: lane l the dims 4l .. 4l+3 of both gradients
            for (int kr = warp; kr < NKV; kr += 8) {
                if (kv0 + kr >= T) break;
                float4 v4, k4;
                asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                             : "=f"(v4.x), "=f"(v4.y), "=f"(v4.z), "=f"(v4.w)
                             : "r"(sdv + kr * 512 + lane * 16));
                asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                             : "=f"(k4.x), "=f"(k4.y), "=f"(k4.z), "=f"(k4.w)
                             : "r"(sdk + kr * 512 + lane * 16));
                const size_t off = (head_rows + kv0 + kr) * kD + 4 * lane;
                write_grad4(a, off, v4, k4);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace ssa
