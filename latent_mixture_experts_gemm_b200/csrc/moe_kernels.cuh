// moe_kernels.cuh -- the non-tensor-core steps of the LatentMoE layer forward:
// top-K' routing with renormalised softmax, the counting sort of (token, slot)
// pairs by expert, and the fixed-order combine.
#pragma once
#include <cfloat>
#include <climits>
#include "ptx.cuh"

namespace lmoe {

// The non-template kernels below have internal linkage (static) so that more
// than one translation unit of the library can include this header.

// Workspace header words (int32), written on the device.
enum : int {
    HDR_ERR = 0,        // device error bits
    HDR_ROWS = 1,       // R: (token, slot) pairs routed to FFN experts
    HDR_MT = 2,         // entries of the tensor-core M-tile list
    HDR_NSMALL = 3,     // entries of the weight-streaming list
    HDR_EP_BAD = 4,     // 1: the received counts of the expert-parallel experts stage were rejected
    HDR_PT = 5,         // entries of the CTA-pair tile list (the same experts as the M-tile list, 256-row entries)
    HDR_WORDS = 16,
};

// ============================================================================ routing
// One warp per token.  Scores are the router logits plus the optional bias;
// the K' largest are selected (value descending, expert id ascending on ties)
// and their softmax is renormalised over the selection:
//   w_k = exp(l_k - l_max) / sum_{j in S} exp(l_j - l_max).
// Lane j holds experts j, j+32, ... as order-preserving 32-bit keys.
//   1. The K'-th largest key tau is found bit by bit from the top: keep a bit
//      when at least K' keys are >= the prefix with it (counts by redux.sync).
//   2. All keys > tau are selected; among keys == tau the lowest ids fill the
//      remaining slots (ballots in id order).
//   3. The K' selected (key, id) pairs are compacted to lanes 0..K'-1 and put in
//      slot order by a warp bitonic sort on (key descending, id ascending).
// Every step is exact integer work on the keys: no floating-point comparison
// other than the fp32 values the keys encode.

// Order-preserving map of an fp32 value to an unsigned key (larger value, larger key).
__device__ __forceinline__ uint32_t order_key(float v) {
    const uint32_t u = __float_as_uint(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// (key, id) a precedes b: larger key first, then lower id.
__device__ __forceinline__ bool slot_before(uint32_t ka, uint32_t ia, uint32_t kb, uint32_t ib) {
    return ka > kb || (ka == kb && ia < ib);
}

// One compare-exchange step of a warp bitonic network on (key, id) pairs in
// slot order (larger key first, then lower id); `e` is the element's index in
// the sequence, `size` the bitonic block length, `stride` the partner distance.
__device__ __forceinline__ void bitonic_step(uint32_t& k, uint32_t& i, int e, int size, int stride, int lane) {
    const uint32_t ok = __shfl_xor_sync(0xffffffffu, k, stride);
    const uint32_t oi = __shfl_xor_sync(0xffffffffu, i, stride);
    const bool lower = (lane & stride) == 0;  // this element keeps the earlier slot of the pair
    const bool ascending = (e & size) == 0;   // direction of this bitonic block (slot order)
    const bool mine_first = slot_before(k, i, ok, oi);
    if (lower == ascending ? !mine_first : mine_first) {
        k = ok;
        i = oi;
    }
}

// Top-K' and renormalised softmax of one token, by one warp.  s_key / s_id:
// 64 words each of this warp's shared memory.
//
// Fast path: the K'-th largest of the 32 lane maxima is a lower bound of the
// K'-th largest key (it is the K'-th largest of a subset), so every selected
// key is among the keys at or above it.  When at most 64 keys qualify, they are
// sorted outright (64-element warp bitonic sort) and the first K' are taken.
// Otherwise the exact radix selection below runs.  SMEM_ROW: the logit row is
// in shared memory (plain loads) rather than in global memory written by an
// earlier kernel (read-only-cache loads).
template <int NPL, bool SMEM_ROW = false>
__device__ __forceinline__ void topk_one_token(const float* __restrict__ row, const float* __restrict__ bias,
                                               int n_tot, int K, uint32_t* s_key, uint32_t* s_id,
                                               int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
    const int lane = threadIdx.x & 31;
    const uint32_t below = (1u << lane) - 1u;
    // all loads first, so that they are in flight together (the row sits in L2: one round trip, not NPL)
    float lv[NPL], bv[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        lv[i] = e < n_tot ? (SMEM_ROW ? row[e] : __ldg(row + e)) : 0.0f;
        bv[i] = (bias != nullptr && e < n_tot) ? __ldg(bias + e) : 0.0f;
    }
    uint32_t key[NPL];
    uint32_t lmax = 0;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        key[i] = e < n_tot ? order_key(lv[i] + bv[i]) : 0u;  // 0: no expert
        lmax = max(lmax, key[i]);
    }
    // K'-th largest lane maximum (descending bitonic sort of the 32 maxima by key)
    uint32_t sk = lmax, si = static_cast<uint32_t>(lane);
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) bitonic_step(sk, si, lane, size, stride, lane);
    const uint32_t lb = max(__shfl_sync(0xffffffffu, sk, K - 1), 1u);
    uint32_t cand = 0;
#pragma unroll
    for (int i = 0; i < NPL; ++i)
        if (key[i] >= lb) cand |= 1u << i;
    const int n_cand = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<uint32_t>(__popc(cand))));

    uint32_t mk, mi;
    if (n_cand <= 64) {
        // compact the candidates to 64 slots in id order, then sort them into slot order
        int base = 0;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const uint32_t m = __ballot_sync(0xffffffffu, (cand >> i) & 1u);
            if ((cand >> i) & 1u) {
                const int c = base + __popc(m & below);
                s_key[c] = key[i];
                s_id[c] = static_cast<uint32_t>(lane + 32 * i);
            }
            base += __popc(m);
        }
        __syncwarp();
        uint32_t k0 = lane < n_cand ? s_key[lane] : 0u, i0 = lane < n_cand ? s_id[lane] : 0xffffffffu;
        uint32_t k1 = lane + 32 < n_cand ? s_key[lane + 32] : 0u, i1 = lane + 32 < n_cand ? s_id[lane + 32] : 0xffffffffu;
        __syncwarp();
#pragma unroll
        for (int size = 2; size <= 64; size <<= 1) {
#pragma unroll
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
                if (stride == 32) {  // partner in the same lane: element lane vs lane + 32 (ascending block)
                    if (!slot_before(k0, i0, k1, i1)) {
                        const uint32_t tk = k0, ti = i0;
                        k0 = k1, i0 = i1, k1 = tk, i1 = ti;
                    }
                } else {
                    bitonic_step(k0, i0, lane, size, stride, lane);
                    bitonic_step(k1, i1, lane + 32, size, stride, lane);
                }
            }
        }
        mk = lane < K ? k0 : 0u;
        mi = lane < K ? i0 : 0xffffffffu;
    } else {
        // exact radix selection: tau = the K'-th largest key, bit by bit from the top
        uint32_t tau = 0;
#pragma unroll 1
        for (int b = 31; b >= 0; --b) {
            const uint32_t c2 = tau | (1u << b);
            uint32_t c = 0;
#pragma unroll
            for (int i = 0; i < NPL; ++i) c += key[i] >= c2 ? 1u : 0u;
            if (__reduce_add_sync(0xffffffffu, c) >= static_cast<uint32_t>(K)) tau = c2;
        }
        // keys above tau, then the lowest ids among keys equal to tau
        uint32_t gt = 0;
#pragma unroll
        for (int i = 0; i < NPL; ++i) gt += key[i] > tau ? 1u : 0u;
        const int need = K - static_cast<int>(__reduce_add_sync(0xffffffffu, gt));
        uint32_t sel = 0;
        int before = 0;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const uint32_t tie = __ballot_sync(0xffffffffu, key[i] == tau);
            const int order = before + __popc(tie & below);
            if (key[i] > tau || (key[i] == tau && order < need)) sel |= 1u << i;
            before += __popc(tie);
        }
        int base = 0;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const uint32_t m = __ballot_sync(0xffffffffu, (sel >> i) & 1u);
            if ((sel >> i) & 1u) {
                const int c = base + __popc(m & below);
                s_key[c] = key[i];
                s_id[c] = static_cast<uint32_t>(lane + 32 * i);
            }
            base += __popc(m);
        }
        __syncwarp();
        mk = lane < K ? s_key[lane] : 0u;
        mi = lane < K ? s_id[lane] : 0xffffffffu;
#pragma unroll
        for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
            for (int stride = size >> 1; stride > 0; stride >>= 1) bitonic_step(mk, mi, lane, size, stride, lane);
    }
    const float sel_v = key_value(mk);
    const float vmax = __shfl_sync(0xffffffffu, sel_v, 0);
    const float ex = lane < K ? expf(sel_v - vmax) : 0.0f;
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane < K) {
        idx_out[lane] = static_cast<int32_t>(mi);
        w_out[lane] = ex / sum;
    }
}

template <int NPL>
__global__ void __launch_bounds__(128) topk_softmax_kernel(const float* __restrict__ logits, int ld,
                                                           const float* __restrict__ bias, int T, int n_tot, int K,
                                                           int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
    pdl_begin();
    __shared__ uint32_t s_key[4][64], s_id[4][64];
    const int warp = threadIdx.x >> 5;
    const int t = blockIdx.x * (blockDim.x >> 5) + warp;
    if (t >= T) return;
    topk_one_token<NPL>(logits + static_cast<size_t>(t) * ld, bias, n_tot, K, s_key[warp], s_id[warp],
                        idx_out + static_cast<size_t>(t) * K, w_out + static_cast<size_t>(t) * K);
}

// Few-token router: the in-order sum of the split-K partials, as
// swap_reduce_kernel takes it, with the top-K' selection folded in.  Blocks
// 0 .. T-1 take one token each: its router logits (fp32, also stored), then
// its top-K' and renormalised softmax by one warp on the logits kept in shared
// memory.  The blocks after them take the z columns (bf16), one element per
// thread.  Router GEMM, selection and softmax end in this kernel, with no
// separate top-K' launch.
//   z[t][n] = bf16(sum of partial row n), n < n0
//   logits[t][c] = sum of partial row p1 + c, c < n1
template <int NT, int NPL>
__global__ void __launch_bounds__(512) router_reduce_topk_kernel(const float* __restrict__ partial, int part_rows,
                                                                 int splits, int T, int n0, int n1, int p1,
                                                                 __nv_bfloat16* __restrict__ out0, int ld0,
                                                                 float* __restrict__ logits, int ld1,
                                                                 const float* __restrict__ bias, int K,
                                                                 int32_t* __restrict__ idx_out,
                                                                 float* __restrict__ w_out) {
    pdl_begin();
    extern __shared__ float s_logit[];  // n1 values
    __shared__ uint32_t s_key[64], s_id[64];
    auto reduce = [&](int prow, int t) {  // all split loads in flight together; the sum runs in split order
        float pv[16];
#pragma unroll
        for (int sp = 0; sp < 16; ++sp)
            pv[sp] = sp < splits ? partial[(static_cast<size_t>(sp) * part_rows + prow) * NT + t] : 0.f;
        float v = 0.f;
#pragma unroll
        for (int sp = 0; sp < 16; ++sp)
            if (sp < splits) v += pv[sp];
        return v;
    };
    if (static_cast<int>(blockIdx.x) < T) {
        const int t = blockIdx.x;
        for (int c = threadIdx.x; c < n1; c += blockDim.x) {
            const float v = reduce(p1 + c, t);
            logits[static_cast<size_t>(t) * ld1 + c] = v;
            s_logit[c] = v;
        }
        __syncthreads();
        if (threadIdx.x < 32)
            topk_one_token<NPL, true>(s_logit, bias, n1, K, s_key, s_id, idx_out + static_cast<size_t>(t) * K,
                                      w_out + static_cast<size_t>(t) * K);
    } else {
        const long i = static_cast<long>(blockIdx.x - T) * blockDim.x + threadIdx.x;
        if (i >= static_cast<long>(n0) * T) return;
        const int n = static_cast<int>(i % n0), t = static_cast<int>(i / n0);
        out0[static_cast<size_t>(t) * ld0 + n] = __float2bfloat16_rn(reduce(n, t));
    }
}

// ============================================================================ dispatch
// Stable counting sort of the flat slots i = t*K' + k by expert id, built from
// a presence bitmap: bit (t % 32) of word [t / 32][e] says token t chose e.
// The position of slot (t, k) with expert e is
//   offsets[e] + prefix[t / 32][e] + popcount(word[t / 32][e] below bit t % 32)
// which orders each expert's slots by token, i.e. by i (a token picks an expert
// at most once).  Every step is integer arithmetic: bit-exact and deterministic.

// One warp per 32-token word; 8 words per block.
static __global__ void __launch_bounds__(256) dispatch_bitmap_kernel(const int32_t* __restrict__ idx, int T, int K,
                                                              int n_tot, uint32_t* __restrict__ bitmap,
                                                              int* __restrict__ hdr) {
    pdl_begin();
    extern __shared__ uint32_t sbits[];  // [8][n_tot]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int word = blockIdx.x * 8 + warp;
    const int nwords = (T + 31) >> 5;
    if (word >= nwords) return;
    uint32_t* mine = sbits + warp * n_tot;
    for (int e = lane; e < n_tot; e += 32) mine[e] = 0;
    __syncwarp();
    const int t = word * 32 + lane;
    if (t < T) {
        for (int k = 0; k < K; ++k) {
            const int e = idx[static_cast<size_t>(t) * K + k];
            if (e < 0 || e >= n_tot) {
                atomicOr(&hdr[HDR_ERR], DEVERR_BAD_INDEX);
                continue;
            }
            // only this lane sets its bit: finding it set means this token named e before
            if (atomicOr(&mine[e], 1u << lane) & (1u << lane)) atomicOr(&hdr[HDR_ERR], DEVERR_REPEATED_INDEX);
        }
    }
    __syncwarp();
    for (int e = lane; e < n_tot; e += 32) bitmap[static_cast<size_t>(word) * n_tot + e] = mine[e];
}

// One warp per expert: exclusive prefix of per-word counts and the total.
static __global__ void __launch_bounds__(256) dispatch_expert_scan_kernel(const uint32_t* __restrict__ bitmap, int T,
                                                                   int n_tot, uint32_t* __restrict__ prefix,
                                                                   int* __restrict__ counts) {
    pdl_begin();
    const int lane = threadIdx.x & 31;
    const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (e >= n_tot) return;
    const int nwords = (T + 31) >> 5;
    int running = 0;
    for (int base = 0; base < nwords; base += 32) {
        const int w = base + lane;
        const int c = w < nwords ? __popc(bitmap[static_cast<size_t>(w) * n_tot + e]) : 0;
        int incl = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += o;
        }
        if (w < nwords) prefix[static_cast<size_t>(w) * n_tot + e] = running + incl - c;
        running += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) counts[e] = running;
}

// Exclusive scan over a block of up to 1024 threads.  `scratch` holds 33 ints.
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = (blockDim.x + 31) >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int s = lane < nwarps ? scratch[lane] : 0;
        int si = s;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, si, off);
            if (lane >= off) si += o;
        }
        scratch[lane] = si - s;
        if (lane == 31) scratch[32] = si;
    }
    __syncthreads();
    const int out = scratch[warp] + incl - v;
    *total = scratch[32];
    __syncthreads();
    return out;
}

// Offsets (exclusive scan of counts), the tensor-core M-tile list (experts
// with more than `small_max` rows, split in 128-row tiles), the CTA-pair tile
// list (the same experts in entries of up to 256 rows) and the
// weight-streaming list (experts with 1..small_max rows).  A negative
// small_max selects chunk mode instead (block-scaled experts, which only
// stream): every FFN expert with rows enters the weight-streaming list as
// entries of at most -small_max rows each, and the M-tile list stays empty.
// Body for a single block of 1024 threads, thread e holding expert e's row
// count c (0 for e >= n_tot); returns offsets[e].

// Weight-streaming list entries of expert e with c rows starting at sorted row off.
__device__ __forceinline__ int stream_entries(bool ffn, int c, int small_max) {
    if (!ffn || c <= 0) return 0;
    if (small_max < 0) return (c - small_max - 1) / (-small_max);
    return c <= small_max ? 1 : 0;
}
__device__ __forceinline__ void write_stream_entries(int4* __restrict__ small_list, int pos, int n, int e, int off,
                                                     int c, int small_max) {
    const int chunk = small_max < 0 ? -small_max : c;
    for (int i = 0; i < n; ++i) small_list[pos + i] = make_int4(e, off + chunk * i, min(chunk, c - chunk * i), 0);
}
// CTA-pair list entries of expert e (c rows from sorted row off): 256 rows each, the rest last.
__device__ __forceinline__ void write_pair_entries(int4* __restrict__ pt_list, int pos, int n, int e, int off, int c) {
    for (int i = 0; i < n; ++i) pt_list[pos + i] = make_int4(e, off + 256 * i, min(256, c - 256 * i), 0);
}

__device__ __forceinline__ int offsets_and_tiles(int c, int n_tot, int n_ffn, int small_max, int* __restrict__ offsets,
                                                 int4* __restrict__ mt_list, int4* __restrict__ small_list,
                                                 int4* __restrict__ pt_list, int* __restrict__ hdr, int* scratch) {
    const int e = threadIdx.x;
    int total;
    const int off = block_exclusive_scan(c, scratch, &total);
    if (e < n_tot) offsets[e] = off;
    if (e == 0) offsets[n_tot] = total;
    const bool ffn = e < n_ffn;
    const bool tc = ffn && small_max >= 0 && c > small_max;
    const int ntile = tc ? (c + 127) / 128 : 0;
    const int ptile = tc ? (c + 255) / 256 : 0;
    const int small = stream_entries(ffn, c, small_max);
    int mt_total, small_total, pt_total;
    const int mt_pos = block_exclusive_scan(ntile, scratch, &mt_total);
    const int sm_pos = block_exclusive_scan(small, scratch, &small_total);
    const int pt_pos = block_exclusive_scan(ptile, scratch, &pt_total);
    for (int i = 0; i < ntile; ++i) mt_list[mt_pos + i] = make_int4(e, off + 128 * i, min(128, c - 128 * i), 0);
    write_pair_entries(pt_list, pt_pos, ptile, e, off, c);
    write_stream_entries(small_list, sm_pos, small, e, off, c, small_max);
    // R = rows of FFN experts = offsets[n_ffn] (FFN ids come first)
    const int ffn_rows_part = ffn ? c : 0;
    int rows_total;
    block_exclusive_scan(ffn_rows_part, scratch, &rows_total);
    if (e == 0) {
        hdr[HDR_ROWS] = rows_total;
        hdr[HDR_MT] = mt_total;
        hdr[HDR_NSMALL] = small_total;
        hdr[HDR_PT] = pt_total;
    }
    return off;
}

// The same as a kernel of one block of 1024 threads, over counts[] in memory.
static __global__ void __launch_bounds__(1024) dispatch_offsets_kernel(const int* __restrict__ counts, int n_tot, int n_ffn,
                                                                int small_max, int* __restrict__ offsets,
                                                                int4* __restrict__ mt_list, int4* __restrict__ small_list,
                                                                int4* __restrict__ pt_list, int* __restrict__ hdr) {
    pdl_begin();
    __shared__ int scratch[33];
    const int e = threadIdx.x;
    offsets_and_tiles(e < n_tot ? counts[e] : 0, n_tot, n_ffn, small_max, offsets, mt_list, small_list, pt_list, hdr,
                      scratch);
}

// Small batches (T <= 256): bitmap, per-expert prefix, offsets, tile lists and
// the placement (perm / inv) in one block of 1024 threads, the bitmap in shared
// memory.  The same positions as the multi-kernel path:
//   pos = offsets[e] + prefix[w][e] + popcount(bits[w][e] below bit t % 32).
constexpr int SMALL_BATCH_WORDS = 8;

// Body of the small-batch dispatch for a block of 1024 threads.  `sm` holds
// (2 * nwords + 1) * n_tot words of dynamic shared memory; `scratch` 33 ints.
__device__ __forceinline__ void dispatch_small_body(const int32_t* __restrict__ idx, int T, int K, int n_tot,
                                                    int n_ffn, int small_max, int* __restrict__ counts,
                                                    int* __restrict__ offsets, int4* __restrict__ mt_list,
                                                    int4* __restrict__ small_list, int4* __restrict__ pt_list,
                                                    int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                                    int* __restrict__ hdr, uint32_t* sm, int* scratch) {
    const int nwords = (T + 31) >> 5;
    uint32_t* bits = sm;
    uint32_t* prefix = sm + nwords * n_tot;
    int* base = reinterpret_cast<int*>(prefix + nwords * n_tot);
    for (int i = threadIdx.x; i < nwords * n_tot; i += blockDim.x) bits[i] = 0;
    __syncthreads();
    const int slots = T * K;
    for (int i = threadIdx.x; i < slots; i += blockDim.x) {
        const int e = idx[i];
        const int t = i / K;
        if (e < 0 || e >= n_tot) {
            atomicOr(&hdr[HDR_ERR], DEVERR_BAD_INDEX);
            continue;
        }
        const uint32_t bit = 1u << (t & 31);  // set by token t's slots only: found set, t named e twice
        if (atomicOr(&bits[(t >> 5) * n_tot + e], bit) & bit) atomicOr(&hdr[HDR_ERR], DEVERR_REPEATED_INDEX);
    }
    __syncthreads();
    const int e = threadIdx.x;
    int c = 0;
    if (e < n_tot)
        for (int w = 0; w < nwords; ++w) {
            prefix[w * n_tot + e] = c;
            c += __popc(bits[w * n_tot + e]);
        }
    int total;
    const int off = block_exclusive_scan(c, scratch, &total);
    if (e < n_tot) {
        counts[e] = c;
        offsets[e] = off;
        base[e] = off;
    }
    if (e == 0) offsets[n_tot] = total;
    const bool ffn = e < n_ffn;
    const bool tc = ffn && small_max >= 0 && c > small_max;
    const int ntile = tc ? (c + 127) / 128 : 0;
    const int ptile = tc ? (c + 255) / 256 : 0;
    const int small = stream_entries(ffn, c, small_max);
    int mt_total, small_total, rows_total, pt_total;
    const int mt_pos = block_exclusive_scan(ntile, scratch, &mt_total);
    const int sm_pos = block_exclusive_scan(small, scratch, &small_total);
    const int pt_pos = block_exclusive_scan(ptile, scratch, &pt_total);
    block_exclusive_scan(ffn ? c : 0, scratch, &rows_total);
    for (int i = 0; i < ntile; ++i) mt_list[mt_pos + i] = make_int4(e, off + 128 * i, min(128, c - 128 * i), 0);
    write_pair_entries(pt_list, pt_pos, ptile, e, off, c);
    write_stream_entries(small_list, sm_pos, small, e, off, c, small_max);
    if (e == 0) {
        hdr[HDR_ROWS] = rows_total;
        hdr[HDR_MT] = mt_total;
        hdr[HDR_NSMALL] = small_total;
        hdr[HDR_PT] = pt_total;
    }
    __syncthreads();  // base[] visible to every thread
    for (int i = threadIdx.x; i < slots; i += blockDim.x) {
        const int ex = idx[i];
        if (ex < 0 || ex >= n_tot) continue;
        const int t = i / K, w = t >> 5;
        const int cell = w * n_tot + ex;
        const int pos = base[ex] + static_cast<int>(prefix[cell]) + __popc(bits[cell] & ((1u << (t & 31)) - 1u));
        perm[pos] = i;
        inv[i] = pos;
    }
}

static __global__ void __launch_bounds__(1024) dispatch_small_kernel(const int32_t* __restrict__ idx, int T, int K, int n_tot,
                                                              int n_ffn, int small_max, int* __restrict__ counts,
                                                              int* __restrict__ offsets, int4* __restrict__ mt_list,
                                                              int4* __restrict__ small_list, int4* __restrict__ pt_list,
                                                              int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                                              int* __restrict__ hdr) {
    pdl_begin();
    extern __shared__ uint32_t sm[];
    __shared__ int scratch[33];
    dispatch_small_body(idx, T, K, n_tot, n_ffn, small_max, counts, offsets, mt_list, small_list, pt_list, perm, inv,
                        hdr, sm, scratch);
}

// One warp per slot: copy the token's feature row to its sorted row (FFN experts only).
static __global__ void __launch_bounds__(256) dispatch_gather_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ inv,
                                                              int T, int K, int n_ffn,
                                                              const __nv_bfloat16* __restrict__ feat, int ld_feat,
                                                              int fdim, __nv_bfloat16* __restrict__ rows_out,
                                                              int ld_rows) {
    pdl_begin();
    const int lane = threadIdx.x & 31;
    const long i = static_cast<long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (i >= static_cast<long>(T) * K) return;
    const int e = idx[i];
    if (e < 0 || e >= n_ffn) return;
    const int t = static_cast<int>(i / K);
    const uint4* src = reinterpret_cast<const uint4*>(feat + static_cast<size_t>(t) * ld_feat);
    uint4* dst = reinterpret_cast<uint4*>(rows_out + static_cast<size_t>(inv[i]) * ld_rows);
    for (int c = lane; c < fdim / 8; c += 32) dst[c] = src[c];
}

// One warp per slot: place it (perm / inv) and, for FFN experts, copy the
// token's feature row (latent z, or x for the standard MoE) to its sorted row.
static __global__ void __launch_bounds__(256) dispatch_scatter_kernel(const int32_t* __restrict__ idx, int T, int K, int n_tot,
                                                               int n_ffn, const uint32_t* __restrict__ bitmap,
                                                               const uint32_t* __restrict__ prefix,
                                                               const int* __restrict__ offsets,
                                                               const __nv_bfloat16* __restrict__ feat, int ld_feat,
                                                               int fdim, __nv_bfloat16* __restrict__ rows_out,
                                                               int ld_rows, int32_t* __restrict__ perm,
                                                               int32_t* __restrict__ inv) {
    pdl_begin();
    const int lane = threadIdx.x & 31;
    const long i = static_cast<long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (i >= static_cast<long>(T) * K) return;
    const int t = static_cast<int>(i / K);
    const int e = idx[i];
    if (e < 0 || e >= n_tot) return;  // flagged by the bitmap kernel
    const int w = t >> 5, b = t & 31;
    const size_t cell = static_cast<size_t>(w) * n_tot + e;
    const int pos = offsets[e] + static_cast<int>(prefix[cell]) + __popc(bitmap[cell] & ((1u << b) - 1u));
    if (lane == 0) {
        perm[pos] = static_cast<int32_t>(i);
        inv[i] = pos;
    }
    if (e < n_ffn) {
        const uint4* src = reinterpret_cast<const uint4*>(feat + static_cast<size_t>(t) * ld_feat);
        uint4* dst = reinterpret_cast<uint4*>(rows_out + static_cast<size_t>(pos) * ld_rows);
        for (int c = lane; c < fdim / 8; c += 32) dst[c] = src[c];
    }
}

// One warp per token (SCATTER_WARPS per block): the token's feature row is read once into shared memory, and
// each of its slots is placed (perm / inv) and, for FFN experts, receives the row at its sorted position by
// one bulk copy from shared memory, so the row is read from memory once instead of once per slot.  The same
// positions as dispatch_scatter_kernel.  Dynamic shared memory: SCATTER_WARPS * fdim * 2 bytes.
constexpr int SCATTER_WARPS = 4;
static __global__ void __launch_bounds__(32 * SCATTER_WARPS) dispatch_scatter_rows_kernel(
    const int32_t* __restrict__ idx, int T, int K, int n_tot, int n_ffn, const uint32_t* __restrict__ bitmap,
    const uint32_t* __restrict__ prefix, const int* __restrict__ offsets, const __nv_bfloat16* __restrict__ feat,
    int ld_feat, int fdim, __nv_bfloat16* __restrict__ rows_out, int ld_rows, int32_t* __restrict__ perm,
    int32_t* __restrict__ inv) {
    pdl_begin();
    extern __shared__ uint4 srow[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t = blockIdx.x * SCATTER_WARPS + warp;
    if (t >= T) return;
    uint4* row = srow + static_cast<size_t>(warp) * (fdim / 8);
    const uint4* src = reinterpret_cast<const uint4*>(feat + static_cast<size_t>(t) * ld_feat);
    for (int c = lane; c < fdim / 8; c += 32) row[c] = src[c];
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the row, visible to the bulk copies
    __syncwarp();
    const int w = t >> 5, b = t & 31;
    for (int k = lane; k < K; k += 32) {
        const long i = static_cast<long>(t) * K + k;
        const int e = idx[i];
        if (e < 0 || e >= n_tot) continue;  // flagged by the bitmap kernel
        const size_t cell = static_cast<size_t>(w) * n_tot + e;
        const int pos = offsets[e] + static_cast<int>(prefix[cell]) + __popc(bitmap[cell] & ((1u << b) - 1u));
        perm[pos] = static_cast<int32_t>(i);
        inv[i] = pos;
        if (e < n_ffn) bulk_store(rows_out + static_cast<size_t>(pos) * ld_rows, row, static_cast<uint32_t>(fdim) * 2);
    }
    bulk_commit();
    bulk_wait_all();  // the copies have read the shared row and written the rows before the warp exits
}

// Experts with at most this many rows take the weight-streaming (swap-AB) GEMM.
constexpr int SMALL_MAX = 32;

// ============================================================================ wait self-test
// One thread waits, with the same bounded wait every kernel of the layer uses,
// on an mbarrier that nothing ever arrives on: after `timeout_ns` it must give
// up, set the timeout bit in `err` and return (no trap, no hang).
static __global__ void wait_selftest_kernel(int* err, unsigned long long timeout_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, &abort_flag, err, timeout_ns);
}

// ============================================================================ combine
// yl_t = sum_k w_tk * o_k in slot order (fp32), o_k the expert's output row, 0
// (zero expert), the token's own feature row (copy expert) or the constant
// vector; plus the residual when the layer has no up-projection.  One block per
// token, 8 columns (16 bytes) per thread per step; no atomics.  The slot table
// (source row, weight) is resolved once per token in shared memory so that the
// K' row loads of a step are independent and issue back to back; a zero expert
// contributes with weight 0 (adding +-0 leaves the fp32 sum unchanged).
template <int UNROLL>
__global__ void __launch_bounds__(128) combine_kernel(
    const __nv_bfloat16* __restrict__ O, int ld_o, const int32_t* __restrict__ inv, const int32_t* __restrict__ idx,
    const float* __restrict__ w, const __nv_bfloat16* __restrict__ feat, int ld_feat,
    const __nv_bfloat16* __restrict__ const_vecs, int T, int K, int L, int n_ffn, int n_zero, int n_copy,
    const __nv_bfloat16* __restrict__ resid, int ld_resid, __nv_bfloat16* __restrict__ out, int ld_out) {
    pdl_begin();
    __shared__ const __nv_bfloat16* s_src[32];
    __shared__ float s_w[32];
    const int t = blockIdx.x;
    if (threadIdx.x < K) {
        const size_t i = static_cast<size_t>(t) * K + threadIdx.x;
        const int e = idx[i];
        const __nv_bfloat16* src = feat + static_cast<size_t>(t) * ld_feat;  // copy expert (and zero: weight 0)
        float wk = w[i];
        if (e < n_ffn) src = O + static_cast<size_t>(inv[i]) * ld_o;
        else if (e < n_ffn + n_zero) wk = 0.0f;
        else if (e >= n_ffn + n_zero + n_copy) src = const_vecs + static_cast<size_t>(e - n_ffn - n_zero - n_copy) * L;
        s_src[threadIdx.x] = src;
        s_w[threadIdx.x] = wk;
    }
    __syncthreads();
    for (int c8 = threadIdx.x; c8 < L / 8; c8 += blockDim.x) {
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = 0.f;
        // UNROLL slot rows are loaded before their FMAs (all K' <= 32 of them for small
        // batches, where latency rules; fewer, for more resident blocks, for large
        // batches, where bandwidth does); the sum always runs in slot order
        for (int k0 = 0; k0 < K; k0 += UNROLL) {
        uint4 rowv[UNROLL];
#pragma unroll
        for (int k = 0; k < UNROLL; ++k)
            if (k0 + k < K) rowv[k] = *reinterpret_cast<const uint4*>(s_src[k0 + k] + c8 * 8);
#pragma unroll
        for (int k = 0; k < UNROLL; ++k) {
            if (k0 + k >= K) break;
            const uint4 v = rowv[k];
            const float wk = s_w[k0 + k];
            acc[0] = fmaf(wk, bf16lo(v.x), acc[0]);
            acc[1] = fmaf(wk, bf16hi(v.x), acc[1]);
            acc[2] = fmaf(wk, bf16lo(v.y), acc[2]);
            acc[3] = fmaf(wk, bf16hi(v.y), acc[3]);
            acc[4] = fmaf(wk, bf16lo(v.z), acc[4]);
            acc[5] = fmaf(wk, bf16hi(v.z), acc[5]);
            acc[6] = fmaf(wk, bf16lo(v.w), acc[6]);
            acc[7] = fmaf(wk, bf16hi(v.w), acc[7]);
        }
        }
        if (resid != nullptr) {
            const uint4 r = *reinterpret_cast<const uint4*>(resid + static_cast<size_t>(t) * ld_resid + c8 * 8);
            acc[0] += bf16lo(r.x); acc[1] += bf16hi(r.x); acc[2] += bf16lo(r.y); acc[3] += bf16hi(r.y);
            acc[4] += bf16lo(r.z); acc[5] += bf16hi(r.z); acc[6] += bf16lo(r.w); acc[7] += bf16hi(r.w);
        }
        *reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * ld_out + c8 * 8) =
            make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                       pack_bf16x2(acc[6], acc[7]));
    }
}

}  // namespace lmoe
