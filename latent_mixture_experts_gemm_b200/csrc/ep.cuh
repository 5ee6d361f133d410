// ep.cuh -- the expert side of expert parallelism.  A rank receives its rows as
// one block per source rank, each block sorted by local expert (the sender's
// counting sort orders rows by global expert id, so by destination rank first).
// The grouped expert GEMMs want each expert's rows together, so the received
// rows are regrouped expert-major before the GEMMs and put back in received
// order after them.  Segment j = s * n_local + e holds source s's rows for
// local expert e.
#pragma once
#include "moe_kernels.cuh"

namespace lmoe {

// One block of 1024 threads, one thread per segment and per local expert
// (n_seg = ep * n_local <= 1024).  From recv_counts [ep][n_local]:
//   * per local expert, its rows (summed over the sources), the offsets and
//     the tile lists, built as the counting sort builds them;
//   * per segment, its first row in the received buffer (src_off: exclusive
//     scan in source-major order; src_off[n_seg] = total) and in the
//     expert-major buffer (dst_base = offsets[e] + the rows of e from the
//     sources before s).
// Counts that are negative, above n_recv, that do not add up to n_recv, or that
// give an expert more than rows_bound rows are rejected: every count is taken
// as 0 (empty tile lists), HDR_EP_BAD is set for the regroup kernels and
// DEVERR_BAD_COUNTS is reported.
static __global__ void __launch_bounds__(1024) ep_prep_kernel(const int32_t* __restrict__ recv_counts, int ep,
                                                              int n_local, int n_recv, int rows_bound, int small_max,
                                                              int* __restrict__ counts, int* __restrict__ offsets,
                                                              int4* __restrict__ mt_list, int4* __restrict__ small_list,
                                                              int4* __restrict__ pt_list,
                                                              int* __restrict__ src_off, int* __restrict__ dst_base,
                                                              int* __restrict__ hdr) {
    pdl_begin();
    __shared__ int s_cnt[1024];
    __shared__ int s_off[1024];
    __shared__ int scratch[33];
    __shared__ long long s_total;
    const int n_seg = ep * n_local;
    const int j = threadIdx.x;
    int cj = j < n_seg ? recv_counts[j] : 0;
    bool bad = cj < 0 || cj > n_recv;
    if (bad) cj = 0;
    s_cnt[j] = cj;
    __syncthreads();
    if (j < 32) {  // 64-bit total: inconsistent counts must not wrap around
        long long t = 0;
        for (int q = j; q < n_seg; q += 32) t += s_cnt[q];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        if (j == 0) s_total = t;
    }
    long long c64 = 0;
    if (j < n_local)
        for (int s = 0; s < ep; ++s) c64 += s_cnt[s * n_local + j];
    bad |= c64 > rows_bound;
    __syncthreads();
    bad |= s_total != static_cast<long long>(n_recv);
    const bool reject = __syncthreads_or(bad) != 0;
    if (reject) {
        cj = 0;
        c64 = 0;
        s_cnt[j] = 0;
    }
    const int c = static_cast<int>(c64);
    if (j < n_local) counts[j] = c;
    const int off =
        offsets_and_tiles(c, n_local, n_local, small_max, offsets, mt_list, small_list, pt_list, hdr, scratch);
    s_off[j] = off;
    int total;
    const int so = block_exclusive_scan(cj, scratch, &total);  // synchronises: s_off and s_cnt are visible
    if (j < n_seg) {
        const int s = j / n_local, e = j - s * n_local;
        int base = s_off[e];
        for (int q = 0; q < s; ++q) base += s_cnt[q * n_local + e];
        src_off[j] = so;
        dst_base[j] = base;
    }
    if (j == 0) {
        src_off[n_seg] = total;
        hdr[HDR_EP_BAD] = reject ? 1 : 0;
        if (reject) atomicOr(&hdr[HDR_ERR], DEVERR_BAD_COUNTS);
    }
}

// Rows per block of the two regroup kernels: one warp per row, 8 warps.
constexpr int EP_ROWS_PER_PASS = 8;

// Received row i of segment j (src_off[j] <= i < src_off[j+1]) goes to row
// dst_base[j] + i - src_off[j] of the expert-major buffer; map[i] keeps that
// row for the way back.  Warps stride over the rows; each block first stages
// the segment table in shared memory ((2 * n_seg + 1) ints).
static __global__ void __launch_bounds__(256) ep_regroup_kernel(const __nv_bfloat16* __restrict__ recv, int n_recv,
                                                                int L, const int* __restrict__ src_off,
                                                                const int* __restrict__ dst_base, int n_seg,
                                                                const int* __restrict__ hdr,
                                                                __nv_bfloat16* __restrict__ rows,
                                                                int32_t* __restrict__ map) {
    pdl_begin();
    extern __shared__ int s_seg[];
    if (hdr[HDR_EP_BAD] != 0) return;
    int* s_src = s_seg;
    int* s_dst = s_seg + n_seg + 1;
    for (int q = threadIdx.x; q <= n_seg; q += blockDim.x) s_src[q] = src_off[q];
    for (int q = threadIdx.x; q < n_seg; q += blockDim.x) s_dst[q] = dst_base[q];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int stride = gridDim.x * EP_ROWS_PER_PASS;
    for (int i = blockIdx.x * EP_ROWS_PER_PASS + (threadIdx.x >> 5); i < n_recv; i += stride) {
        int lo = 0, hi = n_seg - 1;  // largest j with src_off[j] <= i: the non-empty segment holding i
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_src[mid] <= i) lo = mid;
            else hi = mid - 1;
        }
        const int dest = s_dst[lo] + (i - s_src[lo]);
        const uint4* src = reinterpret_cast<const uint4*>(recv + static_cast<size_t>(i) * L);
        uint4* dst = reinterpret_cast<uint4*>(rows + static_cast<size_t>(dest) * L);
        for (int c = lane; c < L / 8; c += 32) dst[c] = src[c];
        if (lane == 0) map[i] = dest;
    }
}

// out[i] = rows[map[i]]: the expert outputs back in received order.
static __global__ void __launch_bounds__(256) ep_unregroup_kernel(const __nv_bfloat16* __restrict__ rows,
                                                                  const int32_t* __restrict__ map, int n_recv, int L,
                                                                  const int* __restrict__ hdr,
                                                                  __nv_bfloat16* __restrict__ out) {
    pdl_begin();
    if (hdr[HDR_EP_BAD] != 0) return;
    const int lane = threadIdx.x & 31;
    const int stride = gridDim.x * EP_ROWS_PER_PASS;
    for (int i = blockIdx.x * EP_ROWS_PER_PASS + (threadIdx.x >> 5); i < n_recv; i += stride) {
        const uint4* src = reinterpret_cast<const uint4*>(rows + static_cast<size_t>(map[i]) * L);
        uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(i) * L);
        for (int c = lane; c < L / 8; c += 32) dst[c] = src[c];
    }
}

}  // namespace lmoe
