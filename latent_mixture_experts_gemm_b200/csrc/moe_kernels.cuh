// moe_kernels.cuh -- the non-tensor-core steps of the LatentMoE layer forward:
// top-K' routing with renormalised softmax, the counting sort of (token, slot)
// pairs by expert, the decode-regime expert weight streaming, and the
// fixed-order combine.
#pragma once
#include <cfloat>
#include <climits>
#include "ptx.cuh"

namespace lmoe {

// Workspace header words (int32), written on the device.
enum : int {
    HDR_ERR = 0,        // device error bits
    HDR_ROWS = 1,       // R: (token, slot) pairs routed to FFN experts
    HDR_MT = 2,         // entries of the tensor-core M-tile list
    HDR_NSMALL = 3,     // entries of the weight-streaming list
    HDR_WORDS = 16,
};

// ============================================================================ routing
// One warp per token.  Scores are the router logits plus the optional bias;
// the K' largest are selected in order (value descending, id ascending on
// ties) by K' rounds of a warp arg-max, and their softmax is renormalised over
// the selection: w_k = exp(l_k - l_max) / sum_j exp(l_j - l_max).
template <int NPL>
__global__ void __launch_bounds__(256) topk_softmax_kernel(const float* __restrict__ logits, int ld,
                                                           const float* __restrict__ bias, int T, int n_tot, int K,
                                                           int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float* row = logits + static_cast<size_t>(t) * ld;
    float v[NPL];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        if (e < n_tot) {
            v[i] = row[e] + (bias != nullptr ? bias[e] : 0.0f);
        } else {
            v[i] = -FLT_MAX;
            taken |= 1u << i;
        }
    }
    float sel_v = -FLT_MAX;
    int sel_e = 0;
#pragma unroll 1
    for (int k = 0; k < K; ++k) {
        float bv = -FLT_MAX;
        int be = INT_MAX;
#pragma unroll
        for (int i = 0; i < NPL; ++i)
            if (!((taken >> i) & 1u) && (be == INT_MAX || v[i] > bv)) {
                bv = v[i];
                be = lane + 32 * i;
            }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            if (oe != INT_MAX && (be == INT_MAX || ov > bv || (ov == bv && oe < be))) {
                bv = ov;
                be = oe;
            }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == k) {
            sel_v = bv;
            sel_e = be;
        }
    }
    const float vmax = __shfl_sync(0xffffffffu, sel_v, 0);
    const float ex = lane < K ? expf(sel_v - vmax) : 0.0f;
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane < K) {
        idx_out[static_cast<size_t>(t) * K + lane] = sel_e;
        w_out[static_cast<size_t>(t) * K + lane] = ex / sum;
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
__global__ void __launch_bounds__(256) dispatch_bitmap_kernel(const int32_t* __restrict__ idx, int T, int K,
                                                              int n_tot, uint32_t* __restrict__ bitmap,
                                                              int* __restrict__ hdr) {
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
            atomicOr(&mine[e], 1u << lane);
        }
    }
    __syncwarp();
    for (int e = lane; e < n_tot; e += 32) bitmap[static_cast<size_t>(word) * n_tot + e] = mine[e];
}

// One warp per expert: exclusive prefix of per-word counts and the total.
__global__ void __launch_bounds__(256) dispatch_expert_scan_kernel(const uint32_t* __restrict__ bitmap, int T,
                                                                   int n_tot, uint32_t* __restrict__ prefix,
                                                                   int* __restrict__ counts) {
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

// Single block of 1024 threads: offsets (exclusive scan of counts), the
// tensor-core M-tile list (experts with more than `small_max` rows, split in
// 128-row tiles) and the weight-streaming list (experts with 1..small_max rows).
__global__ void __launch_bounds__(1024) dispatch_offsets_kernel(const int* __restrict__ counts, int n_tot, int n_ffn,
                                                                int small_max, int* __restrict__ offsets,
                                                                int4* __restrict__ mt_list, int4* __restrict__ small_list,
                                                                int* __restrict__ hdr) {
    __shared__ int scratch[33];
    const int e = threadIdx.x;
    const int c = e < n_tot ? counts[e] : 0;
    int total;
    const int off = block_exclusive_scan(c, scratch, &total);
    if (e < n_tot) offsets[e] = off;
    if (e == 0) offsets[n_tot] = total;
    const bool ffn = e < n_ffn;
    const int ntile = (ffn && c > small_max) ? (c + 127) / 128 : 0;
    const int small = (ffn && c > 0 && c <= small_max) ? 1 : 0;
    int mt_total, small_total;
    const int mt_pos = block_exclusive_scan(ntile, scratch, &mt_total);
    const int sm_pos = block_exclusive_scan(small, scratch, &small_total);
    for (int i = 0; i < ntile; ++i) mt_list[mt_pos + i] = make_int4(e, off + 128 * i, min(128, c - 128 * i), 0);
    if (small) small_list[sm_pos] = make_int4(e, off, c, 0);
    // R = rows of FFN experts = offsets[n_ffn] (FFN ids come first)
    const int ffn_rows_part = ffn ? c : 0;
    int rows_total;
    block_exclusive_scan(ffn_rows_part, scratch, &rows_total);
    if (e == 0) {
        hdr[HDR_ROWS] = rows_total;
        hdr[HDR_MT] = mt_total;
        hdr[HDR_NSMALL] = small_total;
    }
}

// One warp per slot: place it (perm / inv) and, for FFN experts, copy the
// token's feature row (latent z, or x for the standard MoE) to its sorted row.
__global__ void __launch_bounds__(256) dispatch_scatter_kernel(const int32_t* __restrict__ idx, int T, int K, int n_tot,
                                                               int n_ffn, const uint32_t* __restrict__ bitmap,
                                                               const uint32_t* __restrict__ prefix,
                                                               const int* __restrict__ offsets,
                                                               const __nv_bfloat16* __restrict__ feat, int ld_feat,
                                                               int fdim, __nv_bfloat16* __restrict__ rows_out,
                                                               int ld_rows, int32_t* __restrict__ perm,
                                                               int32_t* __restrict__ inv) {
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

// ============================================================================ decode experts
// Experts that received only a few rows (decode) are bound by reading their
// weights once.  Each work item is (list entry, block of 64 output columns);
// a warp covers 8 columns with 4 lanes per column, streaming the weight rows
// with 16-byte loads; the expert's rows (<= SMALL_MAX) sit in shared memory as
// fp32, K in chunks of KCHUNK.  Accumulation is fp32 in a fixed order.
constexpr int SMALL_MAX = 8;
constexpr int GEMV_KCHUNK = 1024;
constexpr int GEMV_THREADS = 256;
constexpr int GEMV_COLS = 64;
enum : int { GEMV_NONE = 0, GEMV_RELU2 = 1, GEMV_SWIGLU = 2 };

template <int ACT>
__global__ void __launch_bounds__(GEMV_THREADS) expert_stream_kernel(
    const __nv_bfloat16* __restrict__ A, int ld_a, const __nv_bfloat16* __restrict__ W, int w_rows_per_expert,
    int up_offset, int K, int n_out, __nv_bfloat16* __restrict__ out, int ld_out, const int4* __restrict__ list,
    const int* __restrict__ list_count) {
    __shared__ __align__(16) float sA[SMALL_MAX * GEMV_KCHUNK];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = lane & 3;
    const int nblk = n_out / GEMV_COLS;
    const int total = (*list_count) * nblk;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        const int j = item / nblk, nb = item % nblk;
        const int4 L = list[j];
        const int e = L.x, row0 = L.y, rows = L.z;
        const int col = nb * GEMV_COLS + warp * 8 + (lane >> 2);
        const __nv_bfloat16* wrow = W + (static_cast<size_t>(e) * w_rows_per_expert + col) * K;
        const __nv_bfloat16* wrow2 = wrow + static_cast<size_t>(up_offset) * K;
        float acc[SMALL_MAX], acc2[SMALL_MAX];
#pragma unroll
        for (int r = 0; r < SMALL_MAX; ++r) acc[r] = 0.f, acc2[r] = 0.f;
        for (int k0 = 0; k0 < K; k0 += GEMV_KCHUNK) {
            const int klen = min(GEMV_KCHUNK, K - k0);
            __syncthreads();
            for (int x = threadIdx.x; x < rows * (klen / 8); x += GEMV_THREADS) {
                const int r = x / (klen / 8), c8 = x % (klen / 8);
                const uint4 v = *reinterpret_cast<const uint4*>(A + static_cast<size_t>(row0 + r) * ld_a + k0 + c8 * 8);
                float4* d = reinterpret_cast<float4*>(sA + r * GEMV_KCHUNK + c8 * 8);
                d[0] = make_float4(bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y));
                d[1] = make_float4(bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w));
            }
            __syncthreads();
#pragma unroll 4
            for (int c = q; c < klen / 8; c += 4) {
                const uint4 wv = ld_stream_v4(wrow + k0 + c * 8);
                const float w0 = bf16lo(wv.x), w1 = bf16hi(wv.x), w2 = bf16lo(wv.y), w3 = bf16hi(wv.y);
                const float w4 = bf16lo(wv.z), w5 = bf16hi(wv.z), w6 = bf16lo(wv.w), w7 = bf16hi(wv.w);
                float u0 = 0, u1 = 0, u2 = 0, u3 = 0, u4 = 0, u5 = 0, u6 = 0, u7 = 0;
                if (ACT == GEMV_SWIGLU) {
                    const uint4 uv = ld_stream_v4(wrow2 + k0 + c * 8);
                    u0 = bf16lo(uv.x), u1 = bf16hi(uv.x), u2 = bf16lo(uv.y), u3 = bf16hi(uv.y);
                    u4 = bf16lo(uv.z), u5 = bf16hi(uv.z), u6 = bf16lo(uv.w), u7 = bf16hi(uv.w);
                }
#pragma unroll
                for (int r = 0; r < SMALL_MAX; ++r) {
                    if (r < rows) {
                        const float4 a0 = *reinterpret_cast<const float4*>(sA + r * GEMV_KCHUNK + c * 8);
                        const float4 a1 = *reinterpret_cast<const float4*>(sA + r * GEMV_KCHUNK + c * 8 + 4);
                        float s = acc[r];
                        s = fmaf(w0, a0.x, s); s = fmaf(w1, a0.y, s); s = fmaf(w2, a0.z, s); s = fmaf(w3, a0.w, s);
                        s = fmaf(w4, a1.x, s); s = fmaf(w5, a1.y, s); s = fmaf(w6, a1.z, s); s = fmaf(w7, a1.w, s);
                        acc[r] = s;
                        if (ACT == GEMV_SWIGLU) {
                            float s2 = acc2[r];
                            s2 = fmaf(u0, a0.x, s2); s2 = fmaf(u1, a0.y, s2); s2 = fmaf(u2, a0.z, s2); s2 = fmaf(u3, a0.w, s2);
                            s2 = fmaf(u4, a1.x, s2); s2 = fmaf(u5, a1.y, s2); s2 = fmaf(u6, a1.z, s2); s2 = fmaf(u7, a1.w, s2);
                            acc2[r] = s2;
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < SMALL_MAX; ++r) {
            acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], 1);
            acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], 2);
            if (ACT == GEMV_SWIGLU) {
                acc2[r] += __shfl_xor_sync(0xffffffffu, acc2[r], 1);
                acc2[r] += __shfl_xor_sync(0xffffffffu, acc2[r], 2);
            }
        }
#pragma unroll
        for (int r = 0; r < SMALL_MAX; ++r) {
            if (r < rows && (r & 3) == q) {
                float v = acc[r];
                if (ACT == GEMV_RELU2) {
                    v = fmaxf(v, 0.f);
                    v = v * v;
                } else if (ACT == GEMV_SWIGLU) {
                    v = v / (1.0f + expf(-v)) * acc2[r];
                }
                out[static_cast<size_t>(row0 + r) * ld_out + col] = __float2bfloat16_rn(v);
            }
        }
    }
}

// ============================================================================ combine
// yl_t = sum_k w_tk * o_k in slot order (fp32), o_k the expert's output row, 0
// (zero expert), the token's own feature row (copy expert) or the constant
// vector; plus the residual when the layer has no up-projection.  One block per
// token, 8 columns (16 bytes) per thread per step; no atomics.
__global__ void __launch_bounds__(128) combine_kernel(
    const __nv_bfloat16* __restrict__ O, int ld_o, const int32_t* __restrict__ inv, const int32_t* __restrict__ idx,
    const float* __restrict__ w, const __nv_bfloat16* __restrict__ feat, int ld_feat,
    const __nv_bfloat16* __restrict__ const_vecs, int T, int K, int L, int n_ffn, int n_zero, int n_copy,
    const __nv_bfloat16* __restrict__ resid, int ld_resid, __nv_bfloat16* __restrict__ out, int ld_out) {
    __shared__ int s_e[32], s_pos[32];
    __shared__ float s_w[32];
    const int t = blockIdx.x;
    if (threadIdx.x < K) {
        const size_t i = static_cast<size_t>(t) * K + threadIdx.x;
        s_e[threadIdx.x] = idx[i];
        s_pos[threadIdx.x] = inv[i];
        s_w[threadIdx.x] = w[i];
    }
    __syncthreads();
    for (int c8 = threadIdx.x; c8 < L / 8; c8 += blockDim.x) {
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = 0.f;
        for (int k = 0; k < K; ++k) {
            const int e = s_e[k];
            const __nv_bfloat16* src;
            if (e < n_ffn) src = O + static_cast<size_t>(s_pos[k]) * ld_o;
            else if (e < n_ffn + n_zero) continue;
            else if (e < n_ffn + n_zero + n_copy) src = feat + static_cast<size_t>(t) * ld_feat;
            else src = const_vecs + static_cast<size_t>(e - n_ffn - n_zero - n_copy) * L;
            const uint4 v = *reinterpret_cast<const uint4*>(src + c8 * 8);
            const float wk = s_w[k];
            acc[0] = fmaf(wk, bf16lo(v.x), acc[0]);
            acc[1] = fmaf(wk, bf16hi(v.x), acc[1]);
            acc[2] = fmaf(wk, bf16lo(v.y), acc[2]);
            acc[3] = fmaf(wk, bf16hi(v.y), acc[3]);
            acc[4] = fmaf(wk, bf16lo(v.z), acc[4]);
            acc[5] = fmaf(wk, bf16hi(v.z), acc[5]);
            acc[6] = fmaf(wk, bf16lo(v.w), acc[6]);
            acc[7] = fmaf(wk, bf16hi(v.w), acc[7]);
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
