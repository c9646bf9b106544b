// Interval form of the skip lists: each row's ascending kept key blocks grouped into maximal
// runs of consecutive indices, (start, length).  The pages describe the per-query-block list
// as the block intervals to compute (summaries of "Accelerating Text-to-Video Generation with
// Calibrated Sparse Attention": [zh] §2.2B, [fr] §2.C) and name mask memory as future work;
// local (band-shaped) masks have long runs, so the interval form is the compact storage of
// the mask dictionary, expanded back to the CSR list the attention kernel walks.
// One warp per row throughout; row offsets by the shared inclusive scan.
#pragma once
#include "ptx.cuh"
#include "select.cuh"

namespace calib {

__device__ __forceinline__ bool run_starts_at(const int16_t* __restrict__ col, int p, int beg, int end) {
    return p < end && (p == beg || col[p] != col[p - 1] + 1);
}

// Encode step 1: runs per row into iv_ptr[row + 1] (iv_ptr[0] = 0).
__global__ void __launch_bounds__(128)
iv_count_kernel(const int32_t* __restrict__ row_ptr, const int16_t* __restrict__ col_idx, int rows,
                int32_t* __restrict__ iv_ptr) {
    const int row = blockIdx.x * (blockDim.x >> 5) + static_cast<int>(warp_id());
    if (row >= rows) return;
    const int lane = static_cast<int>(lane_id());
    const int beg = row_ptr[row], end = row_ptr[row + 1];
    int cnt = 0;
    for (int p0 = beg; p0 < end; p0 += 32) cnt += __popc(__ballot_sync(0xffffffffu, run_starts_at(col_idx, p0 + lane, beg, end)));
    if (lane == 0) {
        iv_ptr[row + 1] = cnt;
        if (row == 0) iv_ptr[0] = 0;
    }
}

// Encode step 3: (start, length) of every run, in row order.
__global__ void __launch_bounds__(128)
iv_fill_kernel(const int32_t* __restrict__ row_ptr, const int16_t* __restrict__ col_idx, int rows,
               const int32_t* __restrict__ iv_ptr, int16_t* __restrict__ iv_start, int16_t* __restrict__ iv_len) {
    const int row = blockIdx.x * (blockDim.x >> 5) + static_cast<int>(warp_id());
    if (row >= rows) return;
    const int lane = static_cast<int>(lane_id());
    const int beg = row_ptr[row], end = row_ptr[row + 1];
    int out = iv_ptr[row];
    for (int p0 = beg; p0 < end; p0 += 32) {
        const int p = p0 + lane;
        const bool s = run_starts_at(col_idx, p, beg, end);
        const uint32_t ball = __ballot_sync(0xffffffffu, s);
        if (s) {
            int q = p + 1;
            while (q < end && col_idx[q] == col_idx[q - 1] + 1) ++q;
            const int idx = out + __popc(ball & lanemask_lt());
            iv_start[idx] = col_idx[p];
            iv_len[idx] = static_cast<int16_t>(q - p);
        }
        out += __popc(ball);
    }
}

// Decode step 1: kept blocks per row (sum of its run lengths) into row_ptr[row + 1].
__global__ void __launch_bounds__(128)
iv_total_kernel(const int32_t* __restrict__ iv_ptr, const int16_t* __restrict__ iv_len, int rows,
                int32_t* __restrict__ row_ptr) {
    const int row = blockIdx.x * (blockDim.x >> 5) + static_cast<int>(warp_id());
    if (row >= rows) return;
    const int lane = static_cast<int>(lane_id());
    int cnt = 0;
    for (int k = iv_ptr[row] + lane; k < iv_ptr[row + 1]; k += 32) cnt += iv_len[k];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    if (lane == 0) {
        row_ptr[row + 1] = cnt;
        if (row == 0) row_ptr[0] = 0;
    }
}

// Decode step 3: expand every run into its block indices.  Each lane takes one run of a
// 32-run chunk; its offset in the row is the exclusive prefix sum of the chunk's lengths.
__global__ void __launch_bounds__(128)
iv_expand_kernel(const int32_t* __restrict__ iv_ptr, const int16_t* __restrict__ iv_start,
                 const int16_t* __restrict__ iv_len, int rows, const int32_t* __restrict__ row_ptr,
                 int16_t* __restrict__ col_idx) {
    const int row = blockIdx.x * (blockDim.x >> 5) + static_cast<int>(warp_id());
    if (row >= rows) return;
    const int lane = static_cast<int>(lane_id());
    const int kb = iv_ptr[row], ke = iv_ptr[row + 1];
    int out = row_ptr[row];
    for (int k0 = kb; k0 < ke; k0 += 32) {
        const int k = k0 + lane;
        const int len = k < ke ? iv_len[k] : 0;
        int incl = len;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        if (k < ke) {
            const int s = iv_start[k];
            const int o = out + incl - len;
            for (int e = 0; e < len; ++e) col_idx[o + e] = static_cast<int16_t>(s + e);
        }
        out += __shfl_sync(0xffffffffu, incl, 31);
    }
}

}  // namespace calib
