// Integer-exact mask selection, cross-input vote, skip-list (CSR) build, load-balancing
// schedule and anchor-row list.  HBM-light kernels: one warp per (head, query block) row.
#pragma once
#include <cstdint>
#include <type_traits>
#include "ptx.cuh"

namespace calib {

constexpr int kSelMaxPerLane = 32;   // nk <= 32 * 32 = 1024 in selection
constexpr int kSelMaxBatch = 256;    // energy matrices per selection call
constexpr int kSelWarps = 4;         // warps per CTA of the selection kernel
constexpr int kSelCompact = 64;      // largest candidate set decided in shared memory
constexpr int kSelBins = 128;        // histogram bins: half exponent levels below the row maximum

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

// Exclusive prefix sum of 64-bit values over the lanes of a warp.
__device__ __forceinline__ uint64_t warp_exclusive_scan_u64(uint64_t v) {
    const uint32_t lane = lane_id();
    uint64_t x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= static_cast<uint32_t>(off)) x += y;
    }
    return x - v;
}

// q = rint(e * 2^shift), ties to even, for e >= 0 given by its binary32 bits x < 2^31,
// computed on the FP64 pipe.  For a normal x (exponent field E >= 1) the binary64 with
// exponent E + 896 + shift and x's significand is exactly e * 2^shift (no overflow or
// underflow for shift in [-86, 200]).  x >> 3 holds E in bits 20..27 above the top 20 bits
// of the significand, so one integer add of (896 + shift) << 20 gives that binary64's high
// word.  A subnormal x is its significand times 2^-149: an exact integer conversion scaled
// by an exact power of two.  Adding 2^52 then rounds the product to an integer, half to
// even (e * 2^shift < 2^52 here), and q is the low 52 bits of the sum.  This is the same
// integer as rounding the significand shifted by E' - 150 + shift bits (E' = max(E, 1))
// with round-half-even on the bits shifted out; a CPU check compared the two on every
// exponent and on exact halves.
template <bool SUBNORMAL = true>
__device__ __forceinline__ uint64_t quantize_energy(uint32_t x, int shift) {
    const uint32_t hi = (x >> 3) + ((896u + static_cast<uint32_t>(shift)) << 20);
    double d = __hiloint2double(static_cast<int>(hi), static_cast<int>(x << 29));
    if constexpr (SUBNORMAL) {
        const uint32_t E = x >> 23;
        // a subnormal x is its significand times 2^-149: an exact integer conversion and an
        // exact scaling by a power of two (built from its exponent field)
        const double ds = __dmul_rn(__uint2double_rn(x & 0x7FFFFFu),
                                    __hiloint2double(static_cast<int>((874u + static_cast<uint32_t>(shift)) << 20), 0));
        d = E ? d : ds;
    }
    const double r = __dadd_rn(d, 4503599627370496.0);            // + 2^52
    return static_cast<uint64_t>(__double_as_longlong(r)) & 0xFFFFFFFFFFFFFull;
}

// Position of word w of a row staged in shared memory: with PAD, 4 words of padding after
// every 32, which keeps 4-word groups aligned and spreads the lanes' runs over the banks.
template <bool PAD>
__device__ __forceinline__ int staged_word(int w) { return PAD ? w + 4 * (w >> 5) : w; }

// Shared-memory reductions by shared-space address (no generic-address check).
// Adds lo at addr and hi at addr + OFF (one base register, an immediate offset).
template <int OFF>
__device__ __forceinline__ void red_shared_add_pair(uint32_t addr, uint32_t lo, uint32_t hi) {
    asm volatile("red.shared.add.u32 [%0], %1;\n\tred.shared.add.u32 [%0+%3], %2;"
                 ::"r"(addr), "r"(lo), "r"(hi), "n"(OFF) : "memory");
}
__device__ __forceinline__ void red_shared_or(uint32_t addr, uint32_t v) {
    asm volatile("red.shared.or.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Minimal tau-energy selection, one warp per (row, chunk of batch entries); lane l holds
// key blocks [l*MPL, (l+1)*MPL) of the row (nk <= 32*MPL).  See calib_select_mask in
// calibatt.h for the rule.  With q_j the row's integer energies (shift chosen so that the
// total stays below 2^53), forced total F and threshold T, the kept set is: the forced
// blocks, every free block with q_j > v, and the first c free blocks (ascending j) with
// q_j == v, where v is the largest value with F + sum_{free, q_j >= v} q_j >= T.
//
// For e >= 0 the binary32 bit pattern b is monotone in e, and q is monotone in e, so with
// G(u) = F + sum_{free, b_j >= u} q_j the largest pattern u* with G(u*) >= T is the pattern
// of a free energy whose q is exactly v (G changes only where an element with q > 0 drops
// out).  u* is found without a search over all the row's values:
//   1. histogram: every free block with q > 0 adds q to the bin of its pattern, bins being
//      half exponent levels counted down from the row's largest free pattern (b >> 22);
//      q > 0 only within 53 levels of the row maximum, so 128 bins hold every such block.
//      The sums are exact: q_j < 2^(52-c) with c = ceil(log2 nk) is split at bit 32-c into
//      a low part (row total < 2^32) and a high part (row total < 2^30), each added with a
//      32-bit shared-memory atomic.
//   2. one warp scan of the 128 bins gives Q, T and the first bin k* (from the top) whose
//      cumulative sum reaches T, so u* lies in bin k*, and A = G(top of bin k*) < T.
//   3. the blocks of bin k* (usually a few: a factor-of-sqrt(2) band of energies) are
//      moved to shared memory in index order, two per lane, and each computes G at its own
//      pattern from the others; u* is the largest pattern with G >= T.
//   4. if no block outside bin k* can have q == v (true where q is exact from the pattern
//      just below the bin up, else checked by quantizing the two patterns just outside the
//      bin), the blocks above bin k* are kept, and the bin's own blocks are decided in
//      shared memory (q > v kept, then ties in index order).
// A row whose bin k* holds more than 64 blocks, or whose ties may cross the bin's edges,
// takes the exact bisection over the bit patterns instead (at most 31 steps over all of the
// row's elements).
template <int MPL>
__global__ void __launch_bounds__(kSelWarps * 32, MPL <= 8 ? 8 : (MPL <= 16 ? 6 : (MPL <= 20 ? 5 : 3)))
select_mask_kernel(const __grid_constant__ SelectParams p) {
    static_assert(MPL >= 1 && MPL <= kSelMaxPerLane, "per-lane count");
    constexpr int NB = kSelBins;
    __shared__ __align__(16) uint32_t hist[kSelWarps][2 * NB];     // low parts, then high parts
    __shared__ __align__(16) uint4 cand[kSelWarps][kSelCompact];   // (b, q low, q high, j)
    __shared__ uint32_t kmask[kSelWarps][32];                      // kept candidates, by j
    // A row of words, for rows that are not 16-byte aligned and for the fallback.  Staged
    // rows place word w at w + 4 * (w / 32) when MPL % 8 == 0: the lanes' 16-byte accesses at
    // a stride of MPL words then fall on distinct banks.
    constexpr bool PAD = MPL % 8 == 0;
    __shared__ __align__(16) uint32_t rowb[kSelWarps][(PAD ? 36 : 32) * MPL];
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
    uint32_t* hlo = hist[wib];
    uint32_t* hhi = hist[wib] + NB;
    reinterpret_cast<uint4*>(hlo)[lane] = make_uint4(0, 0, 0, 0);  // bins 4*lane .. 4*lane+3
    reinterpret_cast<uint4*>(hhi)[lane] = make_uint4(0, 0, 0, 0);
    __syncwarp();

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
            } else {
                // rows not 16-byte aligned: coalesced 4-byte loads into the warp's row buffer,
                // then each lane reads its run back with 16-byte shared loads
                uint32_t* rb = rowb[wib];
#pragma unroll
                for (int k = 0; k < MPL; ++k) {
                    const int j = 32 * k + static_cast<int>(lane);
                    rb[staged_word<PAD>(j)] = j < nk ? __float_as_uint(E[j]) : 0u;
                }
                __syncwarp();
#pragma unroll
                for (int v = 0; v < MPL / 4; ++v) {
                    const uint4 x = *reinterpret_cast<const uint4*>(rb + staged_word<PAD>(j0 + 4 * v));
                    b[4 * v] = x.x;
                    b[4 * v + 1] = x.y;
                    b[4 * v + 2] = x.z;
                    b[4 * v + 3] = x.w;
                }
                __syncwarp();                                // read before the buffer is reused
            }
        } else {
#pragma unroll
            for (int m = 0; m < MPL; ++m) b[m] = j0 + m < nk ? __float_as_uint(E[j0 + m]) : 0u;
        }
        // Patterns below +inf's (0x7F800000) are +0 and the finite positive energies.  Only
        // a warp holding a larger pattern sanitises: negative, NaN or infinite energies
        // count as 0 (and are reported); -0 becomes +0.
        uint32_t xmax = 0;
#pragma unroll
        for (int m = 0; m < MPL; ++m) xmax = b[m] > xmax ? b[m] : xmax;
        if (__any_sync(0xffffffffu, xmax >= 0x7F800000u)) {
            bool bad = false;
            xmax = 0;
#pragma unroll
            for (int m = 0; m < MPL; ++m) {
                const float x = __uint_as_float(b[m]);
                if (!(x >= 0.f) || x == INFINITY) bad = true;
                if (!(x > 0.f) || x == INFINITY) b[m] = 0u;
                xmax = b[m] > xmax ? b[m] : xmax;
            }
            if (__any_sync(0xffffffffu, bad) && lane == 0) raise_status(STATUS_BAD_ENERGY);
        }
        xmax = warp_max_u32(xmax);

        uint32_t kbits = fbits;
        if (xmax == 0u) {
            const int jd = i < nk ? i : 0;                   // all-zero row
            if (jd >= j0 && jd < j0 + MPL) kbits |= 1u << (jd - j0);
        } else {
            const int shift = 52 - float_exponent_p(xmax) - c;
            // forced blocks: their q counts toward F; they are not free (pattern 0)
            uint64_t F = 0;
            uint32_t bmax = xmax;                             // largest free pattern
            if (__any_sync(0xffffffffu, fbits != 0u)) {
                uint32_t fl = 0, fh = 0;
#pragma unroll
                for (int m = 0; m < MPL; ++m) {
                    if ((fbits >> m) & 1u) {
                        const uint64_t q = quantize_energy(b[m], shift);
                        fl += static_cast<uint32_t>(q) & lomask;
                        fh += static_cast<uint32_t>(q >> cs);
                        b[m] = 0u;
                    }
                }
                F = join(warp_sum_u32(fh), warp_sum_u32(fl));
                bmax = 0;
#pragma unroll
                for (int m = 0; m < MPL; ++m) bmax = b[m] > bmax ? b[m] : bmax;
                bmax = warp_max_u32(bmax);
            }
            const uint32_t btop = bmax >> 22;                 // bin 0: the top half level
            // 1. histogram of the free blocks' q by half level below the top
            // Blocks with q > 0 lie within 107 bins of the top; a block further down has q = 0,
            // and clamping its bin to the last one adds nothing there.  It can become a
            // candidate only if the answer lies in that last bin, where its q = 0 keeps it out
            // of the kept set (v > 0).
            // bin d = min(btop - (b >> 22), NB - 1) of a free block (b <= bmax) sits at
            // a_top - 4 * (b >> 22), clamped to the last bin's address
            const uint32_t a_top = smem_u32(hlo) + 4u * btop, a_last = smem_u32(hlo) + 4u * (NB - 1);
            uint32_t bm1 = 0xFFFFFFFFu;                       // smallest free pattern minus 1
#pragma unroll
            for (int m = 0; m < MPL; ++m) bm1 = min(bm1, b[m] - 1u);
            const bool sub = bm1 < 0x7FFFFFu;                 // a subnormal free energy: 1 <= b < 2^23
            auto add_bins = [&](auto subnormal) {
#pragma unroll
                for (int m = 0; m < MPL; ++m) {
                    if (b[m] != 0u) {
                        const uint64_t q = quantize_energy<decltype(subnormal)::value>(b[m], shift);
                        const uint32_t a = min(a_top - 4u * (b[m] >> 22), a_last);
                        red_shared_add_pair<4 * NB>(a, static_cast<uint32_t>(q) & lomask,
                                                    __funnelshift_rc(static_cast<uint32_t>(q),
                                                                     static_cast<uint32_t>(q >> 32), cs));
                    }
                }
            };
            if (__any_sync(0xffffffffu, sub)) add_bins(std::true_type{});
            else add_bins(std::false_type{});
            __syncwarp();
            // 2. scan of the bins (lane l: bins 4l .. 4l+3), clearing them for the next row
            const uint4 lo4 = reinterpret_cast<const uint4*>(hlo)[lane];
            const uint4 hi4 = reinterpret_cast<const uint4*>(hhi)[lane];
            __syncwarp();
            reinterpret_cast<uint4*>(hlo)[lane] = make_uint4(0, 0, 0, 0);
            reinterpret_cast<uint4*>(hhi)[lane] = make_uint4(0, 0, 0, 0);
            const uint64_t s0 = join(hi4.x, lo4.x), s1 = join(hi4.y, lo4.y), s2 = join(hi4.z, lo4.z),
                           s3 = join(hi4.w, lo4.w);
            const uint64_t p0 = s0, p1 = p0 + s1, p2 = p1 + s2, p3 = p2 + s3;   // inclusive, within lane
            const uint64_t base = warp_exclusive_scan_u64(p3);
            const uint64_t Qf = __shfl_sync(0xffffffffu, base + p3, 31);
            const uint64_t Q = F + Qf;
            uint64_t T = __double2ull_rz(ceil(__dmul_rn(p.tau[bi], __ull2double_rn(Q))));
            if (T < 1) T = 1;
            if (F < T) {
                // first bin whose cumulative sum reaches T
                const uint64_t C = F + base;
                const uint64_t gap = C >= T ? 0ull : T - C;   // C + p_k >= T  <=>  p_k >= gap
                const int kl = p0 >= gap ? 0 : (p1 >= gap ? 1 : (p2 >= gap ? 2 : (p3 >= gap ? 3 : 4)));
                const uint32_t has = __ballot_sync(0xffffffffu, kl < 4);   // non-empty: the total reaches T
                const int L = __ffs(has) - 1;
                const int kls = __shfl_sync(0xffffffffu, kl, L);
                const uint64_t Aown = C + (kl == 0 ? 0 : (kl == 1 ? p0 : (kl == 2 ? p1 : p2)));
                const uint64_t A = __shfl_sync(0xffffffffu, Aown, L);        // G(top of bin k*)
                const uint32_t kstar = static_cast<uint32_t>(4 * L + kls);
                // bin k* holds the free patterns in [in_lo, hi_p): the last bin also every
                // pattern below its top, and no bin holds pattern 0 (forced, zero, padding)
                const uint32_t top = btop - kstar;
                const uint32_t lo_p = top << 22, hi_p = (top + 1) << 22;
                const uint32_t in_lo = kstar == static_cast<uint32_t>(NB - 1) ? 1u : (lo_p > 0u ? lo_p : 1u);
                // 3. the blocks of bin k*, in index order
                uint32_t cmask = 0, above = 0;               // this lane's blocks in / above bin k*
#pragma unroll
                for (int m = 0; m < MPL; ++m) {
                    cmask |= (b[m] >= in_lo && b[m] < hi_p ? 1u : 0u) << m;
                    above |= (b[m] >= hi_p ? 1u : 0u) << m;
                }
                const uint32_t cl = __popc(cmask);
                const uint32_t nc = warp_sum_u32(cl);
                bool done = false;
                if (nc <= static_cast<uint32_t>(kSelCompact)) {
                    const uint32_t pos0 = warp_exclusive_scan(cl);
                    uint4* cw = cand[wib];
                    // each block's slot is fixed by the blocks before it (so the slots are in
                    // index order); its q is filled in by the lane that reads the slot
                    uint32_t pos = pos0;
#pragma unroll
                    for (int m = 0; m < MPL; ++m)
                        if ((cmask >> m) & 1u) cw[pos++] = make_uint4(b[m], 0u, 0u, static_cast<uint32_t>(j0 + m));
                    kmask[wib][lane] = 0u;
                    __syncwarp();
                    const bool two = nc > 32;                    // second slot in use (warp-uniform)
                    const bool v0 = lane < nc, v1 = two && lane + 32 < nc;
                    uint4 c0 = v0 ? cw[lane] : make_uint4(0, 0, 0, 0);
                    uint4 c1 = make_uint4(0, 0, 0, 0);
                    if (v0) {
                        const uint64_t q = quantize_energy(c0.x, shift);
                        c0.y = static_cast<uint32_t>(q);
                        c0.z = static_cast<uint32_t>(q >> 32);
                        cw[lane] = c0;
                    }
                    if (two) {
                        if (v1) {
                            c1 = cw[lane + 32];
                            const uint64_t q = quantize_energy(c1.x, shift);
                            c1.y = static_cast<uint32_t>(q);
                            c1.z = static_cast<uint32_t>(q >> 32);
                            cw[lane + 32] = c1;
                        }
                    }
                    __syncwarp();
                    // G at each candidate's own pattern
                    uint64_t G0 = A, G1 = A;
                    // a loop per slot count; at MPL = 16 one loop with the second slot's test
                    // inside measured faster (the two loops change its register allocation)
                    constexpr bool kSplitLoop = MPL != 16;
                    if (!kSplitLoop) {
                        for (uint32_t x = 0; x < nc; ++x) {
                            const uint4 e = cw[x];
                            const uint64_t qe = (static_cast<uint64_t>(e.z) << 32) | e.y;
                            if (e.x >= c0.x) G0 += qe;
                            if (two && e.x >= c1.x) G1 += qe;
                        }
                    } else if (two) {
                        for (uint32_t x = 0; x < nc; ++x) {
                            const uint4 e = cw[x];
                            const uint64_t qe = (static_cast<uint64_t>(e.z) << 32) | e.y;
                            if (e.x >= c0.x) G0 += qe;
                            if (e.x >= c1.x) G1 += qe;
                        }
                    } else {
                        for (uint32_t x = 0; x < nc; ++x) {
                            const uint4 e = cw[x];
                            if (e.x >= c0.x) G0 += (static_cast<uint64_t>(e.z) << 32) | e.y;
                        }
                    }
                    const uint32_t ustar =
                        warp_max_u32(max((v0 && G0 >= T) ? c0.x : 0u, (v1 && G1 >= T) ? c1.x : 0u));
                    const uint64_t v = quantize_energy(ustar, shift);       // > 0 (see above)
                    // 4. no block outside bin k* may tie with v.  An energy of exponent field E
                    // (E' = max(E, 1)) is an integer multiple of 2^(E' - 150), so where
                    // E' - 150 + shift >= 0 at the pattern just below the bin, q is the exact
                    // e * 2^shift from there up: distinct patterns give distinct q, and no block
                    // outside the bin ties with v.  Otherwise the two patterns just outside the
                    // bin are quantised.
                    const uint32_t x_lo = lo_p > 0u ? lo_p - 1u : 0u;
                    const bool exact = max(static_cast<int>(x_lo >> 23), 1) - 150 + shift >= 0;
                    const bool straddle = !exact && ((lo_p > 0 && quantize_energy(lo_p - 1, shift) == v) ||
                                                     quantize_energy(hi_p, shift) == v);
                    if (!straddle && v != 0) {
                        const uint64_t q0 = (static_cast<uint64_t>(c0.z) << 32) | c0.y;
                        const bool gt0 = v0 && q0 > v, eq0 = v0 && q0 == v;
                        // the sum of q over the kept candidates, in the histogram's two 32-bit parts
                        uint32_t gl = gt0 ? static_cast<uint32_t>(q0) & lomask : 0u;
                        uint32_t gh = gt0 ? __funnelshift_rc(c0.y, c0.z, cs) : 0u;
                        bool gt1 = false, eq1 = false;
                        if (two) {
                            const uint64_t q1 = (static_cast<uint64_t>(c1.z) << 32) | c1.y;
                            gt1 = v1 && q1 > v;
                            eq1 = v1 && q1 == v;
                            gl += gt1 ? static_cast<uint32_t>(q1) & lomask : 0u;
                            gh += gt1 ? __funnelshift_rc(c1.y, c1.z, cs) : 0u;
                        }
                        const uint64_t R = T - A - join(warp_sum_u32(gh), warp_sum_u32(gl));   // > 0
                        // ties in index order: the tie of rank r is kept iff the r ties before it
                        // leave the sum short of T, r * v < R (the first ceil(R / v) of them)
                        const uint32_t e0 = __ballot_sync(0xffffffffu, eq0);
                        const uint32_t r0 = __popc(e0 & lanemask_lt());
                        const uint32_t km_a = smem_u32(kmask[wib]);
                        if (gt0 || (eq0 && static_cast<uint64_t>(r0) * v < R))
                            red_shared_or(km_a + 4 * (c0.w >> 5), 1u << (c0.w & 31));
                        if (two) {
                            const uint32_t e1 = __ballot_sync(0xffffffffu, eq1);
                            const uint32_t r1 = __popc(e0) + __popc(e1 & lanemask_lt());
                            if (gt1 || (eq1 && static_cast<uint64_t>(r1) * v < R))
                                red_shared_or(km_a + 4 * (c1.w >> 5), 1u << (c1.w & 31));
                        }
                        __syncwarp();
                        // this lane's blocks j0 .. j0 + MPL - 1 lie in at most two mask words,
                        // where only blocks of bin k* have bits
                        const uint32_t w0 = kmask[wib][j0 >> 5];
                        const uint32_t w1 = kmask[wib][min(j0 + MPL - 1, 32 * 32 - 1) >> 5];
                        const uint64_t wins = ((static_cast<uint64_t>(w1) << 32) | w0) >> (j0 & 31);
                        const uint32_t lanebits = MPL >= 32 ? 0xFFFFFFFFu : ((1u << MPL) - 1u);
                        kbits |= above | (static_cast<uint32_t>(wins) & lanebits);
                        done = true;
                    }
                    __syncwarp();                                 // candidates read before reuse
                }
                if (!done) {
                    // exact bisection over the bit patterns (rare rows).  The row's free
                    // patterns go to shared memory and the loops below run over it without
                    // unrolling, so this path stays small next to the fast one.
                    uint32_t* rb = rowb[wib];
#pragma unroll
                    for (int m = 0; m < MPL; ++m) rb[j0 + m] = b[m];
                    __syncwarp();
                    auto G_all = [&](uint32_t u) -> uint64_t {   // u >= 1: forced and padding have b = 0
                        uint32_t sl = 0, sh = 0;
#pragma unroll 1
                        for (int x = static_cast<int>(lane); x < 32 * MPL; x += 32) {
                            const uint32_t bx = rb[x];
                            if (bx >= u) {
                                const uint64_t q = quantize_energy(bx, shift);
                                sl += static_cast<uint32_t>(q) & lomask;
                                sh += static_cast<uint32_t>(q >> cs);
                            }
                        }
                        return F + join(warp_sum_u32(sh), warp_sum_u32(sl));
                    };
                    uint32_t ul = 0, uh = bmax + 1;              // G(0) = Q >= T, G(bmax + 1) = F < T
                    while (uh - ul > 1) {
                        const uint32_t mid = ul + ((uh - ul) >> 1);
                        if (G_all(mid) >= T) ul = mid;
                        else uh = mid;
                    }
                    const uint64_t v = quantize_energy(ul, shift);
                    // free blocks above v are kept; ties at v in index order (this lane's
                    // blocks are j0 .. j0 + MPL - 1)
                    uint32_t gl = 0, gh = 0, ce = 0, eqbits = 0;
#pragma unroll 1
                    for (int m = 0; m < MPL; ++m) {
                        const uint32_t bx = rb[j0 + m];              // forced and padding: 0
                        const uint64_t q = bx ? quantize_energy(bx, shift) : 0ull;
                        if (q > v) {
                            kbits |= 1u << m;
                            gl += static_cast<uint32_t>(q) & lomask;
                            gh += static_cast<uint32_t>(q >> cs);
                        } else if (q == v) {
                            eqbits |= 1u << m;
                            ++ce;
                        }
                    }
                    const uint64_t R = T - F - join(warp_sum_u32(gh), warp_sum_u32(gl));   // > 0
                    // exact ceil(R / v): a float estimate, then integer steps (R <= nk * v)
                    uint64_t need = v ? static_cast<uint64_t>(__fdividef(__ull2float_rn(R), __ull2float_rn(v))) : 0ull;
                    if (v) {
                        while (need * v < R) ++need;
                        while (need > 0 && (need - 1) * v >= R) --need;
                    }
                    uint64_t rank = warp_exclusive_scan(ce);
#pragma unroll 1
                    for (int m = 0; m < MPL; ++m) {
                        if ((eqbits >> m) & 1u) {
                            if (rank < need) kbits |= 1u << m;
                            ++rank;
                        }
                    }
                    __syncwarp();                                 // rb read before the next entry
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
                            // bit i of x times 1 + 2^7 + 2^14 + 2^21 lands at bit 8i (the
                            // sixteen products sit at distinct bits: no carries)
                            const uint32_t x = (kbits >> (4 * v)) & 0xFu;
                            reinterpret_cast<uint32_t*>(M + j0)[v] = (x * 0x00204081u) & 0x01010101u;
                        }
                    }
                }
            }
            if constexpr (MPL % 4 == 0 && !PAD) {
                if (!p.vec) {
                    // rows not 4-byte aligned, at MPL = 4 or 20 (an odd number of words per
                    // lane, so the lanes' word stores fall on distinct banks): the lane's mask
                    // bytes go to the row buffer, then the warp stores the row with coalesced
                    // byte stores.  At the other widths the lanes' own byte stores measured
                    // faster.
                    uint32_t* rb = rowb[wib];
#pragma unroll
                    for (int v = 0; v < MPL / 4; ++v)
                        rb[(j0 >> 2) + v] = (((kbits >> (4 * v)) & 0xFu) * 0x00204081u) & 0x01010101u;
                    __syncwarp();
                    const uint8_t* rbb = reinterpret_cast<const uint8_t*>(rb);
#pragma unroll
                    for (int k = 0; k < MPL; ++k) {
                        const int j = 32 * k + static_cast<int>(lane);
                        if (j < nk) M[j] = rbb[j];
                    }
                    __syncwarp();                            // read before the buffer is reused
                }
            }
            if (!(MPL % 4 == 0) || (PAD && !p.vec)) {
#pragma unroll
                for (int m = 0; m < MPL; ++m)
                    if (j0 + m < nk) M[j0 + m] = static_cast<uint8_t>((kbits >> m) & 1u);
            }
        }
        if (p.count_accum) {
#pragma unroll
            for (int m = 0; m < MPL; ++m) cnt[m >> 2] += ((kbits >> m) & 1u) << (8 * (m & 3));
        }
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
