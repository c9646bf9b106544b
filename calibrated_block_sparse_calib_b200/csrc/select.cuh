// Integer-exact mask selection, cross-input vote, skip-list (CSR) build, load-balancing
// schedule and anchor-row list.  HBM-light kernels: one warp per (head, query block) row.
#pragma once
#include <cstdint>
#include "ptx.cuh"

namespace calib {

constexpr int kSelMaxPerLane = 32;   // nk <= 32 * 32 = 1024 in selection

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}
__device__ __forceinline__ uint64_t warp_sum_u64(uint64_t v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}
__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const uint64_t o = __shfl_xor_sync(0xffffffffu, v, off);
        v = o > v ? o : v;
    }
    return v;
}

// Exponent p with x < 2^p <= 2x for finite x > 0 (the exponent frexp returns), read from
// the IEEE-754 binary32 fields.
__device__ __forceinline__ int float_exponent_p(float x) {
    const uint32_t bits = __float_as_uint(x);
    const int E = static_cast<int>((bits >> 23) & 0xFFu);
    if (E != 0) return E - 126;
    const int msb = 31 - __clz(bits & 0x7FFFFFu);   // subnormal: value = mant * 2^-149
    return msb - 148;
}

// Minimal tau-energy selection, one warp per row, MPL energies per lane (nk <= 32 * MPL).
// See calib_select_mask in calibatt.h for the rule; the kept set is forced blocks, then
// every non-forced block with q_j > v, then the first c non-forced blocks (ascending j)
// with q_j == v, where v is the largest value with F + sum_{q_j >= v} q_j >= T.
//
// v is found by bisection over the binary32 bit patterns b_j of the energies rather than
// over the integer values: for e >= 0 the bit pattern is monotone in e and q_j =
// rint(e_j 2^shift) is monotone in e_j, so with G(u) = F + sum_{free, b_j >= u} q_j the
// largest u with G(u) >= T is the pattern of an energy whose q is exactly v (G steps only
// at element patterns, and a step with q = 0 changes nothing).  That takes at most 31
// steps with 32-bit compares; every sum stays an exact 64-bit integer.
// (16 and 20 energies per lane: six CTAs per SM, trading a few spilled registers for the
// occupancy that hides the bisection's shuffle latency; measured 20% faster at nk = 591)
template <int MPL>
__global__ void __launch_bounds__(128, MPL <= 8 ? 8 : (MPL <= 20 ? 6 : 3))
select_mask_kernel(const float* __restrict__ energy, int rows, int nq, int nk, double tau,
                   const uint8_t* __restrict__ force, uint8_t* __restrict__ mask_out,
                   int32_t* __restrict__ count_accum) {
    static_assert(MPL >= 1 && MPL <= kSelMaxPerLane, "per-lane count");
    const int row = blockIdx.x * (blockDim.x >> 5) + static_cast<int>(warp_id());
    if (row >= rows) return;
    const uint32_t lane = lane_id();
    const int i = row % nq;
    const size_t base = static_cast<size_t>(row) * nk;

    float ev[MPL];
    uint32_t fbits = 0;
    float emax = 0.f;
    bool bad = false;
#pragma unroll
    for (int m = 0; m < MPL; ++m) {
        const int j = static_cast<int>(lane) + 32 * m;
        float x = 0.f;
        if (j < nk) {
            x = energy[base + j];
            if (!(x >= 0.f) || x == INFINITY) { bad = true; x = 0.f; }
            if (force && force[base + j]) fbits |= 1u << m;
        }
        ev[m] = x;
        emax = fmaxf(emax, x);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) emax = fmaxf(emax, __shfl_xor_sync(0xffffffffu, emax, off));
    if (__any_sync(0xffffffffu, bad) && lane == 0) raise_status(STATUS_BAD_ENERGY);

    uint32_t kbits = fbits;
    if (emax > 0.f) {
        const int p = float_exponent_p(emax);
        const int c = nk <= 1 ? 0 : 32 - __clz(nk - 1);
        const int shift = 52 - p - c;                                   // in [-86, 200]
        const double two_shift = __longlong_as_double(static_cast<long long>(shift + 1023) << 52);
        uint64_t q[MPL];
        uint32_t b[MPL];           // bit pattern of a free energy; 0 for forced and padding
        uint64_t Ql = 0, Fl = 0;
        uint32_t bmax = 0;
#pragma unroll
        for (int m = 0; m < MPL; ++m) {
            q[m] = __double2ull_rn(__dmul_rn(static_cast<double>(ev[m]), two_shift));   // exact x 2^shift
            Ql += q[m];
            const bool fr = (fbits >> m) & 1u;
            if (fr) Fl += q[m];
            b[m] = fr ? 0u : __float_as_uint(ev[m]);
            bmax = b[m] > bmax ? b[m] : bmax;
        }
        const uint64_t Q = warp_sum_u64(Ql);
        const uint64_t F = warp_sum_u64(Fl);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const uint32_t o = __shfl_xor_sync(0xffffffffu, bmax, off);
            bmax = o > bmax ? o : bmax;
        }
        uint64_t T = __double2ull_rz(ceil(__dmul_rn(tau, __ull2double_rn(Q))));
        if (T < 1) T = 1;
        if (F < T) {
            // G(0) = Q >= T (forced and padding add 0 at u = 0 only through F), G(bmax + 1) = F < T
            uint32_t lo = 0, hi = bmax + 1;
            constexpr int NACC = MPL < 4 ? MPL : 4;   // independent partial sums: short add chains
            while (hi - lo > 1) {
                const uint32_t mid = lo + ((hi - lo) >> 1);
                uint64_t acc[NACC];
#pragma unroll
                for (int a = 0; a < NACC; ++a) acc[a] = 0;
#pragma unroll
                for (int m = 0; m < MPL; ++m)
                    acc[m % NACC] += b[m] >= mid ? q[m] : 0ull;
                uint64_t sl = acc[0];
#pragma unroll
                for (int a = 1; a < NACC; ++a) sl += acc[a];
                if (F + warp_sum_u64(sl) >= T) lo = mid; else hi = mid;
            }
            // v = q of the free energy whose pattern is lo (it exists and has q > 0)
            uint64_t vl = 0;
#pragma unroll
            for (int m = 0; m < MPL; ++m)
                if (b[m] == lo && !((fbits >> m) & 1u)) vl = q[m] > vl ? q[m] : vl;
            const uint64_t v = warp_max_u64(vl);
            uint64_t gl = 0;
#pragma unroll
            for (int m = 0; m < MPL; ++m)
                if (!((fbits >> m) & 1u) && q[m] > v) { gl += q[m]; kbits |= 1u << m; }
            const uint64_t R = T - F - warp_sum_u64(gl);                 // > 0
            const uint64_t need = (R + v - 1) / v;
            uint64_t taken = 0;
#pragma unroll
            for (int m = 0; m < MPL; ++m) {
                const bool eq = !((fbits >> m) & 1u) && q[m] == v && static_cast<int>(lane) + 32 * m < nk;
                const uint32_t ball = __ballot_sync(0xffffffffu, eq);
                const uint64_t rank = taken + __popc(ball & lanemask_lt());
                if (eq && rank < need) kbits |= 1u << m;
                taken += __popc(ball);
            }
        }
    } else {
        const int jd = i < nk ? i : 0;                                   // all-zero row
        if ((jd & 31) == static_cast<int>(lane)) kbits |= 1u << (jd >> 5);
    }
#pragma unroll
    for (int m = 0; m < MPL; ++m) {
        const int j = static_cast<int>(lane) + 32 * m;
        if (j < nk) {
            const uint8_t k = static_cast<uint8_t>((kbits >> m) & 1u);
            mask_out[base + j] = k;
            if (count_accum) count_accum[base + j] += k;
        }
    }
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
