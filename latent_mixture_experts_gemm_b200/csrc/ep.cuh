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
// Block exchange (block_rows > 0): source s's rows start at s * block_rows,
// src_off holds each segment's first row there, n_recv is the capacity
// ep * block_rows, and the counts of a source must add up to at most
// block_rows instead of the totals adding up to n_recv.
static __global__ void __launch_bounds__(1024) ep_prep_kernel(const int32_t* __restrict__ recv_counts, int ep,
                                                              int n_local, int n_recv, int rows_bound, int small_max,
                                                              int* __restrict__ counts, int* __restrict__ offsets,
                                                              int4* __restrict__ mt_list, int4* __restrict__ small_list,
                                                              int4* __restrict__ pt_list,
                                                              int* __restrict__ src_off, int* __restrict__ dst_base,
                                                              int* __restrict__ hdr, int block_rows) {
    pdl_begin();
    __shared__ int s_cnt[1024];
    __shared__ int s_off[1024];
    __shared__ int s_so[1024];
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
    if (block_rows > 0 && j < ep) {  // each source's rows fit its block
        long long srows = 0;
        for (int e = 0; e < n_local; ++e) srows += s_cnt[j * n_local + e];
        bad |= srows > block_rows;
    }
    __syncthreads();
    if (block_rows == 0) bad |= s_total != static_cast<long long>(n_recv);
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
    s_so[j] = so;
    __syncthreads();
    if (j < n_seg) {
        const int s = j / n_local, e = j - s * n_local;
        int base = s_off[e];
        for (int q = 0; q < s; ++q) base += s_cnt[q * n_local + e];
        // block exchange: the segment's first row in source s's block
        src_off[j] = block_rows > 0 ? s * block_rows + (so - s_so[s * n_local]) : so;
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

// ---------------------------------------------------------------------------- block exchange
// The same exchange with every (source rank, destination rank) pair given a fixed block of block_rows rows:
// the sender's rows for rank r sit at rows r * block_rows .., and rank s's rows arrive at s * block_rows ..
// (the rest of each block is unused).  The split sizes of the all-to-all are then the same for every pair
// and known before the forward, so no count has to reach the host.

// Rank of packed send row i: the largest r with offsets[r * n_local] <= i (the rows are sorted by expert id,
// so rank r's rows are those of experts r * n_local ..).
__device__ __forceinline__ int ep_rank_of_row(const int* __restrict__ offsets, int n_local, int ep, int i) {
    int lo = 0, hi = ep - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (offsets[mid * n_local] <= i) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Packed rows (the counting sort's order) <-> rank blocks, one warp per packed row; to_blocks selects the
// direction.  n_rows is an upper bound on the host; offsets[ep * n_local] is the count on the device.
static __global__ void __launch_bounds__(256) ep_block_copy_kernel(const __nv_bfloat16* __restrict__ src,
                                                                   __nv_bfloat16* __restrict__ dst,
                                                                   const int* __restrict__ offsets, int n_local,
                                                                   int ep, int block_rows, int n_rows, int L,
                                                                   int to_blocks) {
    pdl_begin();
    const int lane = threadIdx.x & 31;
    const int n = min(n_rows, offsets[ep * n_local]);
    const int stride = gridDim.x * EP_ROWS_PER_PASS;
    for (int i = blockIdx.x * EP_ROWS_PER_PASS + (threadIdx.x >> 5); i < n; i += stride) {
        const int r = ep_rank_of_row(offsets, n_local, ep, i);
        const size_t b = static_cast<size_t>(r) * block_rows + (i - offsets[r * n_local]);
        const uint4* s4 = reinterpret_cast<const uint4*>(src + (to_blocks ? static_cast<size_t>(i) : b) * L);
        uint4* d4 = reinterpret_cast<uint4*>(dst + (to_blocks ? b : static_cast<size_t>(i)) * L);
        for (int c = lane; c < L / 8; c += 32) d4[c] = s4[c];
    }
}

// Received rank blocks -> expert-major rows (as ep_regroup_kernel), and back.  Row i of the received buffer
// is row i - s * block_rows of source s's block; it holds a row when that is below source s's count.
// map[i] = its expert-major row, or -1.
static __global__ void __launch_bounds__(256) ep_regroup_blocks_kernel(const __nv_bfloat16* __restrict__ recv,
                                                                       int block_rows, int L,
                                                                       const int32_t* __restrict__ recv_counts,
                                                                       const int* __restrict__ src_off,
                                                                       const int* __restrict__ dst_base, int ep,
                                                                       int n_local, const int* __restrict__ hdr,
                                                                       __nv_bfloat16* __restrict__ rows,
                                                                       int32_t* __restrict__ map) {
    pdl_begin();
    if (hdr[HDR_EP_BAD] != 0) return;
    const int lane = threadIdx.x & 31;
    const int n = ep * block_rows;
    const int stride = gridDim.x * EP_ROWS_PER_PASS;
    for (int i = blockIdx.x * EP_ROWS_PER_PASS + (threadIdx.x >> 5); i < n; i += stride) {
        // the segment of source s holding row i: the last of s's segments that starts at or before i
        const int s = i / block_rows;
        int lo = s * n_local, hi = lo + n_local - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (src_off[mid] <= i) lo = mid;
            else hi = mid - 1;
        }
        const int j = i - src_off[lo];
        const int dest = j < recv_counts[lo] ? dst_base[lo] + j : -1;
        if (lane == 0) map[i] = dest;
        if (dest < 0) continue;
        const uint4* src = reinterpret_cast<const uint4*>(recv + static_cast<size_t>(i) * L);
        uint4* dst = reinterpret_cast<uint4*>(rows + static_cast<size_t>(dest) * L);
        for (int c = lane; c < L / 8; c += 32) dst[c] = src[c];
    }
}

static __global__ void __launch_bounds__(256) ep_unregroup_blocks_kernel(const __nv_bfloat16* __restrict__ rows,
                                                                         const int32_t* __restrict__ map, int n,
                                                                         int L, const int* __restrict__ hdr,
                                                                         __nv_bfloat16* __restrict__ out) {
    pdl_begin();
    if (hdr[HDR_EP_BAD] != 0) return;
    const int lane = threadIdx.x & 31;
    const int stride = gridDim.x * EP_ROWS_PER_PASS;
    for (int i = blockIdx.x * EP_ROWS_PER_PASS + (threadIdx.x >> 5); i < n; i += stride) {
        const int m = map[i];
        if (m < 0) continue;
        const uint4* src = reinterpret_cast<const uint4*>(rows + static_cast<size_t>(m) * L);
        uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(i) * L);
        for (int c = lane; c < L / 8; c += 32) dst[c] = src[c];
    }
}

}  // namespace lmoe
