// Integer-exact mask selection, cross-input vote, skip-list (CSR) build, load-balancing
// schedule and anchor-row list.  HBM-light kernels: one warp per (head, query block) row.
#pragma once
#include <cstdint>
#include "ptx.cuh"

namespace calib {

constexpr int kSelMaxPerLane = 32;   // nk <= 32 * 32 = 1024 in selection
constexpr int kSelMaxBatch = 256;    // energy matrices per selection call
constexpr int kSelWarps = 4;         // warps per CTA of the selection kernel
constexpr int kSelCompact = 64;      // largest candidate set moved to shared memory

// Parameters of one batched selection call.  Batch entry b is the energy matrix
// energy[b] of shape [rows, nk] (rows = H * nq); force_keep and count_accum are shared by
// every entry.
struct SelectParams {
    const float* energy;       // [nb, rows, nk]
    const uint8_t* force;      // [rows, nk] or null
    uint8_t* mask_out;         // [nb, rows, nk] or null
    int32_t* count_accum;      // [rows, nk] or null: += the number of entries keeping (r, j)
    int nb, rows, nq, nk;
    int chunk, n_chunks;       // batch entries per warp; warps per row
    int vec;                   // 1: rows and lane chunks are 16-byte aligned (vector loads)
    double tau[kSelMaxBatch];
};

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}
__device__ __forceinline__ uint32_t warp_sum_u32(uint32_t v) { return __reduce_add_sync(0xffffffffu, v); }
__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) { return __reduce_max_sync(0xffffffffu, v); }
// Exclusive prefix sum over the lanes of a warp.
__device__ __forceinline__ uint32_t warp_exclusive_scan(uint32_t v) {
    const uint32_t lane = lane_id();
    uint32_t x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= static_cast<uint32_t>(off)) x += y;
    }
    return x - v;
}

// Exponent p with x < 2^p <= 2x for finite x > 0 (the exponent frexp returns), read from
// the IEEE-754 binary32 fields.
__device__ __forceinline__ int float_exponent_p(uint32_t bits) {
    const int E = static_cast<int>((bits >> 23) & 0xFFu);
    if (E != 0) return E - 126;
    const int msb = 31 - __clz(bits & 0x7FFFFFu);   // subnormal: value = mant * 2^-149
    return msb - 148;
}

// q = rint(e * 2^shift), ties to even, for e >= 0 given by its binary32 bits x.  The
// significand m and exponent give e = m * 2^(E' - 150) (E' = max(E, 1)), so q = m * 2^k
// with k = E' - 150 + shift: a left shift when k >= 0, else a right shift by s = -k with
// round-half-even on the bits shifted out.  This is the same integer that rounding the
// (exact) binary64 product e * 2^shift gives.
__device__ __forceinline__ uint64_t quantize_bits(uint32_t x, int shift) {
    const uint32_t E = x >> 23;
    const uint32_t m = E ? ((x & 0x7FFFFFu) | 0x800000u) : (x & 0x7FFFFFu);
    const int k = static_cast<int>(E ? E : 1u) - 150 + shift;
    if (k >= 0) return static_cast<uint64_t>(m) << k;
    const int s = -k;
    if (s >= 32) return 0;
    const uint32_t qt = m >> s;
    const uint32_t rem = m & ((1u << s) - 1u);
    const uint32_t half = 1u << (s - 1);
    return qt + ((rem > half || (rem == half && (qt & 1u))) ? 1u : 0u);
}

// Minimal tau-energy selection, one warp per (row, chunk of batch entries); lane l holds
// key blocks [l*MPL, (l+1)*MPL) of the row (nk <= 32*MPL).  See calib_select_mask in
// calibatt.h for the rule.  With q_j the row's integer energies (shift chosen so that the
// total stays below 2^53), forced total F and threshold T, the kept set is: the forced
// blocks, every free block with q_j > v, and the first c free blocks (ascending j) with
// q_j == v, where v is the largest value with F + sum_{free, q_j >= v} q_j >= T.
//
// Finding v.  For e >= 0 the binary32 bit pattern b is monotone in e, and q is monotone in
// e, so with G(u) = F + sum_{free, b_j >= u} q_j the largest pattern u* with G(u*) >= T is
// the pattern of a free energy whose q is exactly v (G changes only where an element with
// q > 0 drops out).  u* is found in two bisections:
//   1. over the exponent field: the largest level e with G(e << 23) >= T (at most 8 steps
//      over all of the row's elements);
//   2. over the 23 low bits inside that level, where only the elements of that level can
//      change G; when they are few (<= 64, the usual case: a factor-of-two band of
//      energies) they are first moved to shared memory, two per lane, so each step
//      touches two values instead of MPL.
// Every sum is exact: q_j < 2^(52-c) with c = ceil(log2 nk) is split at bit 32-c into a
// low part (row total < 2^32) and a high part (row total < 2^30), each reduced over the
// warp with one 32-bit redux.
template <int MPL>
__global__ void __launch_bounds__(kSelWarps * 32, MPL <= 8 ? 8 : (MPL <= 16 ? 6 : (MPL <= 20 ? 5 : 3)))
select_mask_kernel(const __grid_constant__ SelectParams p) {
    static_assert(MPL >= 1 && MPL <= kSelMaxPerLane, "per-lane count");
    __shared__ uint32_t cand_b[kSelWarps][kSelCompact];
    __shared__ uint32_t cand_l[kSelWarps][kSelCompact];
    __shared__ uint32_t cand_h[kSelWarps][kSelCompact];
    const uint32_t wib = warp_id();
    const long long gw = static_cast<long long>(blockIdx.x) * kSelWarps + wib;
    if (gw >= static_cast<long long>(p.rows) * p.n_chunks) return;
    const int row = static_cast<int>(gw % p.rows);
    const int ck = static_cast<int>(gw / p.rows);
    const int bfirst = ck * p.chunk, blast = min(p.nb, bfirst + p.chunk);
    const uint32_t lane = lane_id();
    const int nk = p.nk;
    const int i = row % p.nq;
    const int j0 = static_cast<int>(lane) * MPL;
    const size_t rbase = static_cast<size_t>(row) * nk;
    const int c = nk <= 1 ? 0 : 32 - __clz(nk - 1);
    const int cs = 32 - c;                                   // split bit of q: 22..32
    const uint32_t lomask = cs >= 32 ? 0xFFFFFFFFu : ((1u << cs) - 1u);
    auto join = [&](uint32_t hi_sum, uint32_t lo_sum) -> uint64_t {
        return (static_cast<uint64_t>(hi_sum) << cs) + lo_sum;
    };

    uint32_t fbits = 0;                                      // forced blocks of this row
    if (p.force) {
#pragma unroll
        for (int m = 0; m < MPL; ++m)
            if (j0 + m < nk && p.force[rbase + j0 + m]) fbits |= 1u << m;
    }
    uint32_t cnt[(MPL + 3) / 4];                             // keep counts, one byte per block
#pragma unroll
    for (int w = 0; w < (MPL + 3) / 4; ++w) cnt[w] = 0;

    for (int bi = bfirst; bi < blast; ++bi) {
        const float* E = p.energy + (static_cast<size_t>(bi) * p.rows + row) * nk;
        uint32_t b[MPL];
        if constexpr (MPL % 4 == 0) {
            if (p.vec) {
#pragma unroll
                for (int v = 0; v < MPL / 4; ++v) {
                    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (j0 + 4 * v < nk) x = reinterpret_cast<const float4*>(E + j0)[v];
                    b[4 * v] = __float_as_uint(x.x);
                    b[4 * v + 1] = __float_as_uint(x.y);
                    b[4 * v + 2] = __float_as_uint(x.z);
                    b[4 * v + 3] = __float_as_uint(x.w);
                }
            }
        }
        if (!(MPL % 4 == 0) || !p.vec) {
#pragma unroll
            for (int m = 0; m < MPL; ++m) b[m] = j0 + m < nk ? __float_as_uint(E[j0 + m]) : 0u;
        }
        // negative, NaN or infinite energies count as 0 (and are reported); -0 becomes +0
        bool bad = false;
        uint32_t xmax = 0;
#pragma unroll
        for (int m = 0; m < MPL; ++m) {
            const float x = __uint_as_float(b[m]);
            if (!(x >= 0.f) || x == INFINITY) bad = true;
            if (!(x > 0.f) || x == INFINITY) b[m] = 0u;
            xmax = b[m] > xmax ? b[m] : xmax;
        }
        if (__any_sync(0xffffffffu, bad) && lane == 0) raise_status(STATUS_BAD_ENERGY);
        xmax = warp_max_u32(xmax);

        uint32_t kbits = fbits;
        if (xmax == 0u) {
            const int jd = i < nk ? i : 0;                   // all-zero row
            if (jd >= j0 && jd < j0 + MPL) kbits |= 1u << (jd - j0);
        } else {
            const int shift = 52 - float_exponent_p(xmax) - c;
            uint32_t ql[MPL], qh[MPL];
            uint32_t al = 0, ah = 0, fl = 0, fh = 0, bmax = 0;
#pragma unroll
            for (int m = 0; m < MPL; ++m) {
                const uint64_t q = quantize_bits(b[m], shift);
                ql[m] = static_cast<uint32_t>(q) & lomask;
                qh[m] = static_cast<uint32_t>(q >> cs);
                al += ql[m];
                ah += qh[m];
                if ((fbits >> m) & 1u) {
                    fl += ql[m];
                    fh += qh[m];
                    b[m] = 0u;                               // forced blocks are not free
                }
                bmax = b[m] > bmax ? b[m] : bmax;
            }
            const uint64_t Q = join(warp_sum_u32(ah), warp_sum_u32(al));
            const uint64_t F = join(warp_sum_u32(fh), warp_sum_u32(fl));
            bmax = warp_max_u32(bmax);
            uint64_t T = __double2ull_rz(ceil(__dmul_rn(p.tau[bi], __ull2double_rn(Q))));
            if (T < 1) T = 1;
            if (F < T) {
                // G(u) over every free element of the row (u >= 1: forced and padding have b = 0)
                auto G_all = [&](uint32_t u) -> uint64_t {
                    uint32_t sl = 0, sh = 0;
#pragma unroll
                    for (int m = 0; m < MPL; ++m) {
                        const bool in = b[m] >= u;
                        sl += in ? ql[m] : 0u;
                        sh += in ? qh[m] : 0u;
                    }
                    return F + join(warp_sum_u32(sh), warp_sum_u32(sl));
                };
                // 1. exponent level: G(0) = Q >= T, G((lvl(bmax)+1) << 23) = F < T
                uint32_t lo = 0, hi = (bmax >> 23) + 1;
                uint64_t A = F;                              // G(hi << 23)
                while (hi - lo > 1) {
                    const uint32_t mid = (lo + hi) >> 1;
                    const uint64_t g = G_all(mid << 23);
                    if (g >= T) lo = mid;
                    else { hi = mid; A = g; }
                }
                const uint32_t lvl = lo;
                // 2. low bits inside the level
                uint32_t ul = lvl << 23, uh = (lvl + 1) << 23;
                uint32_t cl = 0;
#pragma unroll
                for (int m = 0; m < MPL; ++m) cl += (b[m] != 0u && (b[m] >> 23) == lvl) ? 1u : 0u;
                const uint32_t nc = warp_sum_u32(cl);
                if (nc <= static_cast<uint32_t>(kSelCompact)) {
                    uint32_t pos = warp_exclusive_scan(cl);
#pragma unroll
                    for (int m = 0; m < MPL; ++m) {
                        if (b[m] != 0u && (b[m] >> 23) == lvl) {
                            cand_b[wib][pos] = b[m];
                            cand_l[wib][pos] = ql[m];
                            cand_h[wib][pos] = qh[m];
                            ++pos;
                        }
                    }
                    __syncwarp();
                    const bool v0 = lane < nc, v1 = lane + 32 < nc;
                    const uint32_t b0 = v0 ? cand_b[wib][lane] : 0u, b1 = v1 ? cand_b[wib][lane + 32] : 0u;
                    const uint32_t l0 = v0 ? cand_l[wib][lane] : 0u, l1 = v1 ? cand_l[wib][lane + 32] : 0u;
                    const uint32_t h0 = v0 ? cand_h[wib][lane] : 0u, h1 = v1 ? cand_h[wib][lane + 32] : 0u;
                    __syncwarp();
                    // G(u) = A + (level elements with b >= u), for u inside the level
                    while (uh - ul > 1) {
                        const uint32_t mid = ul + ((uh - ul) >> 1);
                        const uint32_t sl = (b0 >= mid ? l0 : 0u) + (b1 >= mid ? l1 : 0u);
                        const uint32_t sh = (b0 >= mid ? h0 : 0u) + (b1 >= mid ? h1 : 0u);
                        if (A + join(warp_sum_u32(sh), warp_sum_u32(sl)) >= T) ul = mid;
                        else uh = mid;
                    }
                } else {
                    while (uh - ul > 1) {
                        const uint32_t mid = ul + ((uh - ul) >> 1);
                        if (G_all(mid) >= T) ul = mid;
                        else uh = mid;
                    }
                }
                const uint64_t v = quantize_bits(ul, shift);    // > 0 (see above)
                // free blocks above v are kept; ties at v are taken in index order
                uint32_t gl = 0, gh = 0, ce = 0;
                uint32_t eqbits = 0;
#pragma unroll
                for (int m = 0; m < MPL; ++m) {
                    const uint64_t q = (static_cast<uint64_t>(qh[m]) << cs) | ql[m];
                    const bool fr = !((fbits >> m) & 1u) && j0 + m < nk;
                    if (fr && q > v) {
                        kbits |= 1u << m;
                        gl += ql[m];
                        gh += qh[m];
                    } else if (fr && q == v) {
                        eqbits |= 1u << m;
                        ++ce;
                    }
                }
                const uint64_t R = T - F - join(warp_sum_u32(gh), warp_sum_u32(gl));   // > 0
                uint64_t need = v ? static_cast<uint64_t>(ceil(__ddiv_rn(__ull2double_rn(R), __ull2double_rn(v))))
                                  : 0ull;
                if (v) {
                    while (need * v < R) ++need;                   // exact ceil(R / v)
                    while (need > 0 && (need - 1) * v >= R) --need;
                }
                uint64_t rank = warp_exclusive_scan(ce);
#pragma unroll
                for (int m = 0; m < MPL; ++m) {
                    if ((eqbits >> m) & 1u) {
                        if (rank < need) kbits |= 1u << m;
                        ++rank;
                    }
                }
            }
        }
        if (p.mask_out) {
            uint8_t* M = p.mask_out + (static_cast<size_t>(bi) * p.rows + row) * nk;
            if constexpr (MPL % 4 == 0) {
                if (p.vec) {
#pragma unroll
                    for (int v = 0; v < MPL / 4; ++v) {
                        if (j0 + 4 * v < nk) {
                            const uint32_t x = (kbits >> (4 * v)) & 0xFu;
                            reinterpret_cast<uint32_t*>(M + j0)[v] =
                                (x & 1u) | ((x & 2u) << 7) | ((x & 4u) << 14) | ((x & 8u) << 21);
                        }
                    }
                }
            }
            if (!(MPL % 4 == 0) || !p.vec) {
#pragma unroll
                for (int m = 0; m < MPL; ++m)
                    if (j0 + m < nk) M[j0 + m] = static_cast<uint8_t>((kbits >> m) & 1u);
            }
        }
#pragma unroll
        for (int m = 0; m < MPL; ++m) cnt[m >> 2] += ((kbits >> m) & 1u) << (8 * (m & 3));
    }
    if (p.count_accum) {
#pragma unroll
        for (int m = 0; m < MPL; ++m) {
            const uint32_t k = (cnt[m >> 2] >> (8 * (m & 3))) & 0xFFu;
            if (k && j0 + m < nk) atomicAdd(p.count_accum + rbase + j0 + m, static_cast<int>(k));
        }
    }
}

// Energy-mean aggregation over calibration inputs: mean = sum / n, elementwise, with the
// correctly rounded fp32 division.
__global__ void __launch_bounds__(256)
energy_mean_kernel(const float* __restrict__ sum, long long count, float n, float* __restrict__ mean) {
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    const long long t0 = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const bool vec = ((reinterpret_cast<uintptr_t>(sum) | reinterpret_cast<uintptr_t>(mean)) & 15u) == 0;
    long long done = 0;
    if (vec) {
        const long long n4 = count / 4;
        for (long long x = t0; x < n4; x += stride) {
            const float4 s = reinterpret_cast<const float4*>(sum)[x];
            reinterpret_cast<float4*>(mean)[x] =
                make_float4(__fdiv_rn(s.x, n), __fdiv_rn(s.y, n), __fdiv_rn(s.z, n), __fdiv_rn(s.w, n));
        }
        done = n4 * 4;
    }
    for (long long x = done + t0; x < count; x += stride) mean[x] = __fdiv_rn(sum[x], n);
}

// Cross-input vote, one warp per row: keep iff count * rho_den > rho_num * n_inputs;
// an emptied row keeps its most frequent block (lowest index on ties).
__global__ void __launch_bounds__(128)
aggregate_kernel(const int32_t* __restrict__ counts, int rows, int nk, int n_inputs, int rho_num,
                 int rho_den, uint8_t* __restrict__ mask_out) {
    const int row = blockIdx.x * (blockDim.x >> 5) + static_cast<int>(warp_id());
    if (row >= rows) return;
    const uint32_t lane = lane_id();
    const size_t base = static_cast<size_t>(row) * nk;
    const long long rhs = static_cast<long long>(rho_num) * n_inputs;
    bool any = false;
    int best_c = -1, best_j = 0x7fffffff;
    for (int j0 = 0; j0 < nk; j0 += 32) {
        const int j = j0 + static_cast<int>(lane);
        if (j < nk) {
            const int c = counts[base + j];
            const bool keep = static_cast<long long>(c) * rho_den > rhs;
            any |= keep;
            mask_out[base + j] = keep ? 1 : 0;
            if (c > best_c) { best_c = c; best_j = j; }
        }
    }
    if (__any_sync(0xffffffffu, any)) return;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const int oc = __shfl_xor_sync(0xffffffffu, best_c, off);
        const int oj = __shfl_xor_sync(0xffffffffu, best_j, off);
        if (oc > best_c || (oc == best_c && oj < best_j)) { best_c = oc; best_j = oj; }
    }
    if (lane == 0) mask_out[base + best_j] = 1;
}

// CSR step 1: per-row kept counts into row_ptr[row + 1] (row_ptr[0] = 0).
__global__ void __launch_bounds__(128)
csr_count_kernel(const uint8_t* __restrict__ mask, int rows, int nk, int32_t* __restrict__ row_ptr) {
    const int row = blockIdx.x * (blockDim.x >> 5) + static_cast<int>(warp_id());
    if (row >= rows) return;
    const uint32_t lane = lane_id();
    const size_t base = static_cast<size_t>(row) * nk;
    int cnt = 0;
    for (int j0 = 0; j0 < nk; j0 += 32) {
        const int j = j0 + static_cast<int>(lane);
        cnt += __popc(__ballot_sync(0xffffffffu, j < nk && mask[base + j] != 0));
    }
    if (lane == 0) {
        row_ptr[row + 1] = cnt;
        if (row == 0) row_ptr[0] = 0;
    }
}

// In-place inclusive scan of v[0..n) by one block of 1024 threads (each thread scans a
// contiguous segment, then the segment totals are scanned in shared memory).
__device__ void block_inclusive_scan_inplace(int32_t* v, int n) {
    __shared__ int32_t part[1024];
    const int tid = threadIdx.x, nt = blockDim.x;
    const int seg = (n + nt - 1) / nt;
    const int lo = min(n, tid * seg), hi = min(n, lo + seg);
    int32_t acc = 0;
    for (int x = lo; x < hi; ++x) acc += v[x];
    part[tid] = acc;
    __syncthreads();
    for (int off = 1; off < nt; off <<= 1) {
        const int32_t add = tid >= off ? part[tid - off] : 0;
        __syncthreads();
        part[tid] += add;
        __syncthreads();
    }
    int32_t run = tid > 0 ? part[tid - 1] : 0;
    for (int x = lo; x < hi; ++x) {
        run += v[x];
        v[x] = run;
    }
    __syncthreads();
}

__global__ void __launch_bounds__(1024) csr_scan_kernel(int32_t* row_ptr, int rows) {
    block_inclusive_scan_inplace(row_ptr + 1, rows);
}

// CSR step 3: ascending kept indices of every row.
__global__ void __launch_bounds__(128)
csr_fill_kernel(const uint8_t* __restrict__ mask, int rows, int nk, const int32_t* __restrict__ row_ptr,
                int16_t* __restrict__ col_idx) {
    const int row = blockIdx.x * (blockDim.x >> 5) + static_cast<int>(warp_id());
    if (row >= rows) return;
    const uint32_t lane = lane_id();
    const size_t base = static_cast<size_t>(row) * nk;
    int out = row_ptr[row];
    for (int j0 = 0; j0 < nk; j0 += 32) {
        const int j = j0 + static_cast<int>(lane);
        const bool k = j < nk && mask[base + j] != 0;
        const uint32_t ball = __ballot_sync(0xffffffffu, k);
        if (k) col_idx[out + __popc(ball & lanemask_lt())] = static_cast<int16_t>(j);
        out += __popc(ball);
    }
}

// Schedule: heads in order (so the K/V working set of the CTAs in flight is one or two
// heads and stays in L2), and within a head the query blocks longest-first.  One block of
// 1024 threads per head: a counting sort of the head's rows by kept count (descending),
// stable in row index.  Shared memory: a histogram of 32768 bins.
constexpr int kSchedBins = 32768;
__global__ void __launch_bounds__(1024)
schedule_kernel(const int32_t* __restrict__ row_ptr, int nq, int32_t* __restrict__ work) {
    extern __shared__ int32_t hist[];                // [kSchedBins]
    const int tid = threadIdx.x, nt = blockDim.x;
    const int h = blockIdx.x;
    const int r0 = h * nq;
    for (int b = tid; b < kSchedBins; b += nt) hist[b] = 0;
    __syncthreads();
    for (int r = r0 + tid; r < r0 + nq; r += nt) {
        const int c = min(row_ptr[r + 1] - row_ptr[r], kSchedBins - 1);
        atomicAdd(&hist[kSchedBins - 1 - c], 1);     // bin order = count descending
    }
    __syncthreads();
    // exclusive scan of hist (segments of kSchedBins / 1024 bins per thread)
    {
        __shared__ int32_t part[1024];
        const int seg = kSchedBins / 1024;
        int32_t acc = 0;
        for (int x = tid * seg; x < (tid + 1) * seg; ++x) acc += hist[x];
        part[tid] = acc;
        __syncthreads();
        for (int off = 1; off < nt; off <<= 1) {
            const int32_t add = tid >= off ? part[tid - off] : 0;
            __syncthreads();
            part[tid] += add;
            __syncthreads();
        }
        int32_t run = tid > 0 ? part[tid - 1] : 0;
        for (int x = tid * seg; x < (tid + 1) * seg; ++x) {
            const int32_t v = hist[x];
            hist[x] = run;
            run += v;
        }
    }
    __syncthreads();
    // stable scatter by one warp, rows in index order
    if (tid < 32) {
        const uint32_t lane = lane_id();
        for (int i0 = 0; i0 < nq; i0 += 32) {
            const int i = i0 + static_cast<int>(lane);
            const bool live = i < nq;
            const int r = r0 + i;
            const int bin = live ? kSchedBins - 1 - min(row_ptr[r + 1] - row_ptr[r], kSchedBins - 1) : -1;
            const uint32_t peers = __match_any_sync(0xffffffffu, bin);
            const int leader = __ffs(peers) - 1;
            int basepos = 0;
            if (live && static_cast<int>(lane) == leader) {
                basepos = hist[bin];
                hist[bin] = basepos + __popc(peers);
            }
            basepos = __shfl_sync(0xffffffffu, basepos, leader);
            if (live) work[r0 + basepos + __popc(peers & lanemask_lt())] = (h << 16) | i;
            __syncwarp();
        }
    }
}

// Anchor token indices of a spatial-repetition head (compacted order).
__global__ void anchor_rows_kernel(int F, int Hl, int Wl, int n_text, int stride, int Ar,
                                   int n_anchor, int32_t* __restrict__ rows) {
    const int a = blockIdx.x * blockDim.x + threadIdx.x;
    if (a >= n_anchor) return;
    const int per_frame = Ar * Wl, nva = F * per_frame;
    int t;
    if (a < nva) {
        const int f = a / per_frame, rem = a - f * per_frame;
        const int ya = rem / Wl, x = rem - ya * Wl;
        t = (f * Hl + ya * stride) * Wl + x;
    } else {
        t = F * Hl * Wl + (a - nva);
    }
    rows[a] = t;
}

// Failure-detection self-test: a bounded wait on an mbarrier nothing completes.
__global__ void selftest_wait_kernel(uint64_t timeout_ns) {
    __shared__ __align__(8) uint64_t mbar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(smem_u32(&mbar), 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const WaitCtl ctl{&abort_flag, timeout_ns};
        (void)mbar_wait(smem_u32(&mbar), 0, ctl);
    }
}

}  // namespace calib
