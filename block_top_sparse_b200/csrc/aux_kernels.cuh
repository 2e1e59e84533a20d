// aux_kernels.cuh -- bandwidth-bound helpers of the attention path:
//   * inverse selection index (key block -> list of (query, slot) entries,
//     ascending in query position), built deterministically in three passes,
//     and the launch order of the block-major units (heaviest first);
//   * merge of the block-major sparse forward's per-slot partial outputs;
//   * backward pre/post-processing (D = rowsum(dO o (O + O_lo)), dQ accumulator -> dQ);
//   * bidirectional SmoothL1 alignment loss forward/backward (paper section 5);
//   * dropped attention mass delta = 1 - exp(lse_s - lse_f) (section 4.2).
#pragma once

#include "device.cuh"
#include "pool_select.cuh"

namespace ssa {

constexpr int kIdxChunk = 256;  // queries per counting chunk

// Pass 1: cnt[bh][c][j] = number of entries of block j among queries of chunk c.
__global__ void __launch_bounds__(256) index_count_kernel(const int32_t *__restrict__ idx, int *__restrict__ cnt,
                                                          int T, int k, int nb, int nch) {
    extern __shared__ int hcount[];
    const int bh = blockIdx.y, c = blockIdx.x;
    for (int j = threadIdx.x; j < nb; j += blockDim.x) hcount[j] = 0;
    __syncthreads();
    const int t0 = c * kIdxChunk;
    const int n = min(kIdxChunk, T - t0) * k;
    const int32_t *src = idx + (static_cast<size_t>(bh) * T + t0) * k;
    // 16 loads in flight before their shared-memory atomics (a load after an atomic would wait for it)
    constexpr int U = 16;
    for (int e0 = threadIdx.x; e0 < n; e0 += U * blockDim.x) {
        int jv[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e = e0 + u * blockDim.x;
            jv[u] = e < n ? __ldg(src + e) : -1;
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (jv[u] >= 0 && jv[u] < nb) atomicAdd(&hcount[jv[u]], 1);
    }
    __syncthreads();
    for (int j = threadIdx.x; j < nb; j += blockDim.x) cnt[(static_cast<size_t>(bh) * nch + c) * nb + j] = hcount[j];
}

// Pass 2 (one CTA per head): per-chunk write offsets (in place over cnt),
// list start and length of every block within the head's entry region.
__global__ void __launch_bounds__(1024) index_scan_kernel(int *__restrict__ cnt, int *__restrict__ lstart,
                                                          int *__restrict__ llen, int nb, int nch) {
    __shared__ int warp_tot[32];
    __shared__ int carry;
    const int bh = blockIdx.x;
    int *base = cnt + static_cast<size_t>(bh) * nch * nb;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int j0 = 0; j0 < nb; j0 += blockDim.x) {
        const int j = j0 + threadIdx.x;
        // chunk counts -> exclusive offsets within the block, 16 chunks' loads in flight at a time (a load
        // after a store to the same array would wait for it)
        constexpr int U = 16;
        int total = 0;
        if (j < nb) {
            for (int c0 = 0; c0 < nch; c0 += U) {
                int v[U];
#pragma unroll
                for (int u = 0; u < U; ++u) v[u] = c0 + u < nch ? base[static_cast<size_t>(c0 + u) * nb + j] : 0;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if (c0 + u < nch) base[static_cast<size_t>(c0 + u) * nb + j] = total;
                    total += v[u];
                }
            }
        }
        // exclusive scan over j of the totals rounded up to whole 128-entry tiles
        // (every block's list region starts on a tile boundary)
        const int padded = (total + kListPad - 1) / kListPad * kListPad;
        const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
        int incl = padded;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) warp_tot[w] = incl;
        __syncthreads();
        if (w == 0) {
            int x = (lane < static_cast<int>(blockDim.x >> 5)) ? warp_tot[lane] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += v;
            }
            warp_tot[lane] = x;  // inclusive over warps
        }
        __syncthreads();
        const int start = carry + (w > 0 ? warp_tot[w - 1] : 0) + incl - padded;
        if (j < nb) {
            lstart[bh * nb + j] = start;
            llen[bh * nb + j] = total;
            for (int c0 = 0; c0 < nch; c0 += U) {
                int v[U];
#pragma unroll
                for (int u = 0; u < U; ++u) v[u] = c0 + u < nch ? base[static_cast<size_t>(c0 + u) * nb + j] : 0;
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (c0 + u < nch) base[static_cast<size_t>(c0 + u) * nb + j] = v[u] + start;
            }
        }
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry = start + padded;
        __syncthreads();
    }
}

// Pass 3: one warp per chunk writes entries (t << 8) | slot at their final
// position, in ascending query order (ranks within a 32-query step come from
// lane bitmasks).  k <= 256 and T < 2^23 keep the encoding in an int32.  Each
// 32-query step's selection rows are staged in shared memory by one coalesced
// load (rows padded to k + 1 ints: conflict-free per-lane reads), and the list
// positions (pos, when asked) leave through the same staging, coalesced.
// Shared memory per warp: 2 * nb + 2 * 32 * (k + 1) ints.
__host__ __device__ constexpr size_t index_fill_warp_ints(int nb, int k) {
    return 2 * static_cast<size_t>(nb) + 64 * static_cast<size_t>(k + 1);
}

__global__ void __launch_bounds__(128) index_fill_kernel(const int32_t *__restrict__ idx,
                                                         const int *__restrict__ off, int32_t *__restrict__ entries,
                                                         int32_t *__restrict__ pos, int T, int k, int nb, int nch) {
    extern __shared__ int sm_fill[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, wpc = blockDim.x >> 5;
    const int bh = blockIdx.y, c = blockIdx.x * wpc + warp;
    int *wsm = sm_fill + warp * index_fill_warp_ints(nb, k);
    uint32_t *bits = reinterpret_cast<uint32_t *>(wsm);
    int *run = wsm + nb;
    int *rows = wsm + 2 * nb;              // [32][k + 1] selections of the step's queries
    int *prow = rows + 32 * (k + 1);       // [32][k + 1] their list positions
    if (c < nch) {
        for (int j = lane; j < nb; j += 32) {
            bits[j] = 0u;
            run[j] = off[(static_cast<size_t>(bh) * nch + c) * nb + j];
        }
    }
    __syncwarp();
    if (c >= nch) return;
    int32_t *dst = entries + static_cast<size_t>(bh) * list_stride(T, k, nb);
    const uint32_t lt_mask = (1u << lane) - 1u;
    const int t_end = min(T, (c + 1) * kIdxChunk);
    const int *mine = rows + lane * (k + 1);
    int *mpos = prow + lane * (k + 1);
    for (int tb = c * kIdxChunk; tb < t_end; tb += 32) {
        const int t = tb + lane;
        const size_t base = (static_cast<size_t>(bh) * T + tb) * k;
        const int n = min(32, t_end - tb) * k;  // the step's selections, contiguous in idx
        for (int e = lane; e < 32 * k; e += 32) {
            const int r = e / k;
            rows[r * (k + 1) + (e - r * k)] = e < n ? __ldg(idx + base + e) : -1;
        }
        __syncwarp();
        for (int i = 0; i < k; ++i) {
            const int j = mine[i];
            if (j >= 0 && j < nb) atomicOr(&bits[j], 1u << lane);
        }
        __syncwarp();
        for (int i = 0; i < k; ++i) {
            const int j = mine[i];
            const int at = (j >= 0 && j < nb) ? run[j] + __popc(bits[j] & lt_mask) : -1;
            if (at >= 0) dst[at] = (t << 8) | i;
            mpos[i] = at;
        }
        __syncwarp();
        for (int i = 0; i < k; ++i) {
            const int j = mine[i];
            if (j >= 0 && j < nb) {
                const uint32_t b = bits[j];
                if (b != 0u && lane == __ffs(b) - 1) {
                    run[j] += __popc(b);
                    bits[j] = 0u;
                }
            }
        }
        if (pos) {
            __syncwarp();
            for (int e = lane; e < n; e += 32) {
                const int r = e / k;
                pos[base + e] = prow[r * (k + 1) + (e - r * k)];
            }
        }
        __syncwarp();
    }
}

// Pass 4 (one CTA): launch order of the (head, key block) units of the block-major
// attention kernels.  A unit's work is its number of query tiles, ceil(len / per_tile),
// and the lists are very uneven (early blocks and attention-sink blocks are chosen by
// many queries), so units of at least 5/4 of the mean come first, heaviest first (in
// kOrdHeavy buckets of equal width between the threshold and the maximum); the rest
// follow in head-major order, which keeps the head being worked on in L2.  A stable
// counting sort (ranks from warp match masks, per-warp bucket counts scanned in
// shared memory), so the order is deterministic.
constexpr int kOrdHeavy = 63;            // buckets of heavy units; bucket kOrdHeavy holds the rest
constexpr int kOrdBuckets = kOrdHeavy + 1;

__global__ void __launch_bounds__(1024) unit_order_kernel(const int *__restrict__ llen, int32_t *__restrict__ order,
                                                          int units, int per_tile) {
    __shared__ int wcnt[32][kOrdBuckets];  // per-warp bucket counts of the current chunk, then their offsets
    __shared__ int start[kOrdBuckets];     // running write position of every bucket
    __shared__ unsigned long long red_tot[32];
    __shared__ int red_max[32];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    auto tiles_of = [&](int u) { return (__ldg(llen + u) + per_tile - 1) / per_tile; };
    // total and largest work
    unsigned long long tot = 0;
    int mx = 0;
    for (int u = tid; u < units; u += blockDim.x) {
        const int t = tiles_of(u);
        tot += static_cast<unsigned long long>(t);
        mx = max(mx, t);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        tot += __shfl_xor_sync(0xffffffffu, tot, o);
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (lane == 0) {
        red_tot[warp] = tot;
        red_max[warp] = mx;
    }
    __syncthreads();
    tot = 0;
    mx = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) {
        tot += red_tot[w];
        mx = max(mx, red_max[w]);
    }
    const int thr = max(2, static_cast<int>((5 * tot + 4ull * units - 1) / (4ull * units)));
    auto bucket_of = [&](int u) {
        const int t = tiles_of(u);
        if (t < thr) return kOrdHeavy;
        return mx > thr ? static_cast<int>(static_cast<long long>(mx - t) * (kOrdHeavy - 1) / (mx - thr)) : 0;
    };
    // bucket sizes -> first position of every bucket
    for (int b = tid; b < kOrdBuckets; b += blockDim.x) start[b] = 0;
    __syncthreads();
    for (int u = tid; u < units; u += blockDim.x) atomicAdd(&start[bucket_of(u)], 1);
    __syncthreads();
    if (tid == 0) {
        int acc = 0;
        for (int b = 0; b < kOrdBuckets; ++b) {
            const int c = start[b];
            start[b] = acc;
            acc += c;
        }
    }
    __syncthreads();
    // stable scatter, one unit per thread per chunk
    const int nw = blockDim.x >> 5;
    for (int u0 = 0; u0 < units; u0 += blockDim.x) {
        const int u = u0 + tid;
        const int b = u < units ? bucket_of(u) : -1;
        const unsigned same = __match_any_sync(0xffffffffu, b);
        const int rank = __popc(same & ((1u << lane) - 1u));
        for (int i = lane; i < kOrdBuckets; i += 32) wcnt[warp][i] = 0;
        __syncwarp();
        if (b >= 0 && rank == 0) wcnt[warp][b] = __popc(same);
        __syncthreads();
        for (int i = tid; i < kOrdBuckets; i += blockDim.x) {  // exclusive scan over warps, per bucket
            int acc = start[i];
            for (int w = 0; w < nw; ++w) {
                const int c = wcnt[w][i];
                wcnt[w][i] = acc;
                acc += c;
            }
            start[i] = acc;
        }
        __syncthreads();
        if (b >= 0) order[wcnt[warp][b] + rank] = u;
        __syncthreads();
    }
}

// Merge of the per-slot partials: one warp per query row, 4 columns per lane.
//   lse = log sum_i exp(lse_i),  o = sum_i exp(lse_i - lse) o_i
// The partial of (query, slot i) sits at list position pos[query * k + i] of its
// key head's region (-1: slot not attended), in partial row position * G + (query
// head within the group).  Partials are fp16 (11 significant bits)
// holding o_i * 2^-e_j, where e_j >= 0 is the range exponent of key block
// j = idx[query * k + i] (0 unless |V| in that block reaches 2^15); the word after
// the last block's exponent is non-zero when any exponent is, and only then are
// idx and the exponents read.  For k <= 32 every slot's row is requested as soon as
// the slot positions arrive, before the weights are known.  Lane i holds
// slot i's position and weight (32 slots at a time), so the slots' row loads are
// all in flight at once.  The merged fp32 row is stored as O = bf16(o) and, when
// O_lo is given, O_lo = bf16(o - O).
__device__ __forceinline__ void half4_to_f32(uint2 u, float (&f)[4]) {
    const __half2 a = *reinterpret_cast<const __half2 *>(&u.x), b = *reinterpret_cast<const __half2 *>(&u.y);
    const float2 fa = __half22float2(a), fb = __half22float2(b);
    f[0] = fa.x;
    f[1] = fa.y;
    f[2] = fb.x;
    f[3] = fb.y;
}

template <int NG>  // slot groups of 8 held in registers (k <= 8 * NG); NG = 0: any k, loads after the weights
__global__ void __launch_bounds__(256) sparse_merge_kernel(const int32_t *__restrict__ pos,
                                                           const int32_t *__restrict__ idx,
                                                           const int32_t *__restrict__ bexp,
                                                           const __half *__restrict__ Opart,
                                                           const float *__restrict__ lsepart,
                                                           __nv_bfloat16 *__restrict__ O,
                                                           __nv_bfloat16 *__restrict__ O_lo, float *__restrict__ lse,
                                                           size_t rows, int T, int k, int nb, int G) {
    const size_t row = static_cast<size_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    // query row -> key/value head bh (whose selection, positions and partials it uses), head in group hi
    const size_t qh = row / T, t = row % T;
    const size_t bh = qh / G, hi = qh % G;
    const size_t region = bh * list_stride(T, k, nb);
    const int32_t *ps = pos + (bh * T + t) * k;
    const int32_t *js = idx + (bh * T + t) * k;
    const bool scaled = __ldg(bexp + (rows / T / G) * nb) != 0;
    auto part_row = [&](int p) {  // this lane's 4 columns of the partial at list position p
        return __ldg(reinterpret_cast<const uint2 *>(Opart + ((region + p) * G + hi) * 128) + lane);
    };
    float mx = -INFINITY, wsum = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
    if constexpr (NG > 0) {
        // lane i holds slot i; every slot row is requested before the weights are known
        const int p = lane < k ? __ldg(ps + lane) : -1;
        uint2 u[8 * NG];
#pragma unroll
        for (int q = 0; q < 8 * NG; ++q) {
            const int pq = __shfl_sync(0xffffffffu, p, q);
            u[q] = (q < k && pq >= 0) ? part_row(pq) : make_uint2(0u, 0u);
        }
        const float l = p >= 0 ? __ldg(lsepart + (region + p) * G + hi) : -INFINITY;
        mx = l;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float w = 0.f, wo = 0.f;
        if (p >= 0) {
            w = __expf(l - mx);
            // the partial's weight with its range exponent restored
            wo = scaled ? ldexpf(w, __ldg(bexp + bh * nb + __ldg(js + lane))) : w;
        }
        wsum = w;
#pragma unroll
        for (int q = 0; q < 8 * NG; ++q) {
            const float wq = __shfl_sync(0xffffffffu, wo, q);
            float f[4];
            half4_to_f32(u[q], f);
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[c] = fmaf(wq, f[c], acc[c]);
        }
    } else {
        for (int i0 = 0; i0 < k; i0 += 32) {
            const int p = (i0 + lane < k) ? __ldg(ps + i0 + lane) : -1;
            if (p >= 0) mx = fmaxf(mx, __ldg(lsepart + (region + p) * G + hi));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        for (int i0 = 0; i0 < k; i0 += 32) {
            const int p = (i0 + lane < k) ? __ldg(ps + i0 + lane) : -1;
            float w = 0.f, wo = 0.f;
            if (p >= 0) {
                w = __expf(__ldg(lsepart + (region + p) * G + hi) - mx);
                wo = scaled ? ldexpf(w, __ldg(bexp + bh * nb + __ldg(js + i0 + lane))) : w;
            }
            wsum += w;
            const int n = min(32, k - i0);
            for (int s0 = 0; s0 < n; s0 += 8) {
                uint2 u[8];
                float wu[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int pq = __shfl_sync(0xffffffffu, p, (s0 + q) & 31);
                    wu[q] = __shfl_sync(0xffffffffu, wo, (s0 + q) & 31);
                    u[q] = (s0 + q < n && pq >= 0) ? part_row(pq) : make_uint2(0u, 0u);
                }
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    float f[4];
                    half4_to_f32(u[q], f);
#pragma unroll
                    for (int c = 0; c < 4; ++c) acc[c] = fmaf(wu[q], f[c], acc[c]);
                }
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
    const float inv = 1.f / wsum;
    float o4[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) o4[c] = acc[c] * inv;
    const uint32_t h01 = pack_bf16x2(o4[0], o4[1]), h23 = pack_bf16x2(o4[2], o4[3]);
    reinterpret_cast<uint2 *>(O + row * 128)[lane] = make_uint2(h01, h23);
    if (O_lo) {
        const uint32_t l01 = pack_bf16x2(o4[0] - __uint_as_float(h01 << 16), o4[1] - __uint_as_float(h01 & 0xFFFF0000u));
        const uint32_t l23 = pack_bf16x2(o4[2] - __uint_as_float(h23 << 16), o4[3] - __uint_as_float(h23 & 0xFFFF0000u));
        reinterpret_cast<uint2 *>(O_lo + row * 128)[lane] = make_uint2(l01, l23);
    }
    if (lane == 0) lse[row] = mx + __logf(wsum);
}

// D[row] = sum_c dO[row,c] * (O[row,c] + O_lo[row,c]) (one warp per row; O_lo may be
// NULL); zero the fp32 dQ accumulator row.
template <typename T>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const T *__restrict__ dO, const T *__restrict__ O,
                                                       const T *__restrict__ O_lo, float *__restrict__ Dvec,
                                                       float *__restrict__ dQacc, size_t rows, int d) {
    const size_t row = static_cast<size_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float acc = 0.f;
    for (int c = lane; c < d; c += 32) {
        float o = to_f32(O[row * d + c]);
        if (O_lo) o += to_f32(O_lo[row * d + c]);
        acc += to_f32(dO[row * d + c]) * o;
        if (dQacc) dQacc[row * d + c] = 0.f;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) Dvec[row] = acc;
}

// The same for bf16 rows of d = 128 (the tensor-core path): a warp takes 4 consecutive rows, lane l the
// elements 4l .. 4l+3 of each (8-byte loads), so that the rows' twelve loads are in flight together; the fp32
// accumulator rows are zeroed with 16-byte stores.
constexpr int kPrepRows = 4;  // rows per warp
__global__ void __launch_bounds__(256) bwd_prep_bf16_kernel(const __nv_bfloat16 *__restrict__ dO,
                                                            const __nv_bfloat16 *__restrict__ O,
                                                            const __nv_bfloat16 *__restrict__ O_lo,
                                                            float *__restrict__ Dvec, float *__restrict__ dQacc,
                                                            size_t rows) {
    const size_t row0 = ((static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5) * kPrepRows;
    const int lane = threadIdx.x & 31;
    uint2 g[kPrepRows], o[kPrepRows], lo[kPrepRows];
#pragma unroll
    for (int i = 0; i < kPrepRows; ++i) {
        const size_t row = row0 + i;
        const bool in = row < rows;
        g[i] = in ? __ldg(reinterpret_cast<const uint2 *>(dO + row * 128) + lane) : make_uint2(0u, 0u);
        o[i] = in ? __ldg(reinterpret_cast<const uint2 *>(O + row * 128) + lane) : make_uint2(0u, 0u);
        lo[i] = (in && O_lo) ? __ldg(reinterpret_cast<const uint2 *>(O_lo + row * 128) + lane) : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < kPrepRows; ++i) {
        const uint32_t gw[2] = {g[i].x, g[i].y}, ow[2] = {o[i].x, o[i].y}, lw[2] = {lo[i].x, lo[i].y};
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            acc += __uint_as_float(gw[w] << 16) * (__uint_as_float(ow[w] << 16) + __uint_as_float(lw[w] << 16));
            acc += __uint_as_float(gw[w] & 0xFFFF0000u) *
                   (__uint_as_float(ow[w] & 0xFFFF0000u) + __uint_as_float(lw[w] & 0xFFFF0000u));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        const size_t row = row0 + i;
        if (row < rows) {
            if (lane == 0) Dvec[row] = acc;
            if (dQacc) reinterpret_cast<float4 *>(dQacc + row * 128)[lane] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
}

// out = (accumulate ? out : 0) + acc, rounded once to T.
template <typename T>
__global__ void __launch_bounds__(256) acc_to_out_kernel(const float *__restrict__ acc, T *__restrict__ out,
                                                         size_t n, int accumulate) {
    for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        float v = acc[i];
        if (accumulate) v += to_f32(out[i]);
        if constexpr (sizeof(T) == 2)
            out[i] = __float2bfloat16_rn(v);
        else
            out[i] = v;
    }
}

// ---------------------------------------------------------------------------
// Alignment loss (paper section 5).  Both per-element losses are symmetric, so
// both directions share sum_i l(Of_i - Os_i):
//   loss = (w_sparsity + w_commit) * sum / n
// Pass 1: fixed grid of kAlignBlocks CTAs, per-CTA partial sums (fp32);
// pass 2: one warp adds the partials in fixed order (fp64) -> deterministic.
// ---------------------------------------------------------------------------
constexpr int kAlignBlocks = 1184;  // 8 x 148 SMs

__device__ __forceinline__ float huber(float x, float beta) {
    const float a = fabsf(x);
    return a < beta ? 0.5f * x * x / beta : a - 0.5f * beta;
}

__device__ __forceinline__ float huber_slope(float x, float beta) {
    if (fabsf(x) < beta) return x / beta;
    return x > 0.f ? 1.f : -1.f;
}

// Per-element alignment loss and slope: kind 0 SmoothL1, kind 1 adjusted L2 (0.5 x^2 / beta
// everywhere, the section 7.5 ablation variant).
__device__ __forceinline__ float align_elem(int kind, float x, float beta) {
    return kind ? 0.5f * x * x / beta : huber(x, beta);
}

__device__ __forceinline__ float align_slope(int kind, float x, float beta) {
    return kind ? x / beta : huber_slope(x, beta);
}

template <typename T>
__global__ void __launch_bounds__(256) align_fwd_partial_kernel(const T *__restrict__ Of, const T *__restrict__ Os,
                                                                float *__restrict__ partial, size_t n, int kind,
                                                                float beta) {
    constexpr int V = Vec16<T>::N;
    __shared__ float red[8];
    float acc = 0.f;
    const size_t nv = n / V;
    for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nv;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        float a[V], b[V];
        Vec16<T>::load(Of + i * V, a);
        Vec16<T>::load(Os + i * V, b);
#pragma unroll
        for (int q = 0; q < V; ++q) acc += align_elem(kind, a[q] - b[q], beta);
    }
    if (blockIdx.x == 0)
        for (size_t i = nv * V + threadIdx.x; i < n; i += blockDim.x)
            acc += align_elem(kind, to_f32(Of[i]) - to_f32(Os[i]), beta);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        float s = 0.f;
        for (int w = 0; w < 8; ++w) s += red[w];
        partial[blockIdx.x] = s;
    }
}

__global__ void align_fwd_final_kernel(const float *__restrict__ partial, int nparts, float *__restrict__ loss,
                                       double scale) {
    const int lane = threadIdx.x;
    double s = 0.0;
    for (int i = lane; i < nparts; i += 32) s += partial[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) *loss = static_cast<float>(s * scale);
}

template <typename T>
__global__ void __launch_bounds__(256) align_bwd_kernel(const T *__restrict__ Of, const T *__restrict__ Os,
                                                        const float *__restrict__ dloss, T *__restrict__ dOf,
                                                        T *__restrict__ dOs, size_t n, int kind, float beta,
                                                        float w_s, float w_c, int accumulate) {
    const float g = __ldg(dloss) / static_cast<float>(n);
    const float cf = g * w_s, cs = g * w_c;
    for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const float x = to_f32(Of[i]) - to_f32(Os[i]);
        const float h = align_slope(kind, x, beta);
        float gf = cf * h, gs = -cs * h;  // both slopes are odd: l'(Os - Of) = -l'(Of - Os)
        if (accumulate & 1) gf += to_f32(dOf[i]);
        if (accumulate & 2) gs += to_f32(dOs[i]);
        if constexpr (sizeof(T) == 2) {
            dOf[i] = __float2bfloat16_rn(gf);
            dOs[i] = __float2bfloat16_rn(gs);
        } else {
            dOf[i] = gf;
            dOs[i] = gs;
        }
    }
}

__global__ void __launch_bounds__(256) dropped_mass_kernel(const float *__restrict__ ls, const float *__restrict__ lf,
                                                           float *__restrict__ delta, size_t n) {
    for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x)
        delta[i] = -expm1f(ls[i] - lf[i]);
}

}  // namespace ssa
