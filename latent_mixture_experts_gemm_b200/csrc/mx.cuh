// mx.cuh -- block-scaled (MX) expert weights: encoding and the decode-regime
// weight-streaming GEMM on tcgen05 block-scaled MMAs.
//
// Format (Open Compute Project Microscaling v1.0): blocks of 32 consecutive
// values along the reduction axis K share one E8M0 scale 2^s with
// s = floor(log2 amax) - emax (emax = 8 for E4M3, 2 for E2M1; s clamped to
// [-127, 127], all-zero blocks s = -127).  Each element is value / 2^s
// rounded to nearest even and saturated (448 for E4M3, 6 for E2M1).  The
// pages name MXFP4 as the Kimi K3 serving format (the comparison table of
// "Two Teams, Two Practices"); MXFP8 is the 8-bit member of the same family.
//
// Expert weights are MXFP8 (E4M3) or MXFP4 (E2M1).  The expert GEMMs' token
// operands (the gathered latent rows, and the activation between the two
// expert matrices) are MXFP8.  Both are encoded from the bf16 values this
// library stores.  The MMA applies both operands' block scales
// (kind::mxf8f6f4.block_scale), so the accumulator holds the product of the
// decoded values.
//
// Weight layout in HBM:
//   codes   E4M3: [rows, K] one byte per element.  E2M1: [rows, K/2] two per
//           byte, element 2i in the low nibble of byte i.
//   scales  E8M0 bytes in 512-byte atoms [rows/128][K/128][32][16]: byte
//           (r, c) of atom (R, G) is the scale of row 128R + 32(c/4) + r,
//           block 4G + (c % 4).  This is the layout tcgen05.cp moves into the
//           tensor memory columns the MMA reads its scales from.
// Token-operand layout (workspace): codes [rows, K] bytes; scales
// [rows, K/128, 16] bytes, where chunk g of a row holds the scales of blocks
// 4g .. 4g+3 in its first four bytes (the other twelve are not read).  One
// 16-byte chunk per 128-element stage keeps every scale-factor column the MMA
// reads aligned to four tensor-memory columns.
#pragma once
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "tc_swap.cuh"

namespace lmoe {

// Block scale exponent from the bit pattern of the block's largest magnitude.
__device__ __forceinline__ int mx_scale_exp(uint32_t amax_bits, int emax) {
    if (amax_bits == 0) return -127;
    const int ebits = static_cast<int>(amax_bits >> 23);
    // floor(log2 amax): the exponent field for normals; for subnormals, from the leading one
    const int e = ebits != 0 ? ebits - 127 : (31 - __clz(static_cast<int>(amax_bits))) - 149;
    const int s = e - emax;
    return s < -127 ? -127 : (s > 127 ? 127 : s);
}

// 2^k as a float, k in [-126, 127].
__device__ __forceinline__ float mx_exp2i(int k) { return __uint_as_float(static_cast<uint32_t>(k + 127) << 23); }

__device__ __forceinline__ uint32_t mx_e4m3(float q) {
    return static_cast<uint32_t>(__nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3));
}
__device__ __forceinline__ uint32_t mx_e2m1(float q) {
    return static_cast<uint32_t>(__nv_cvt_float_to_fp4(q, __NV_E2M1, cudaRoundNearest)) & 0xFu;
}

// Encode 32 values (already bf16-exact) in MXFP8; returns the E8M0 byte.
__device__ __forceinline__ uint32_t mx_encode32_e4m3(const float (&v)[32], uint4& lo, uint4& hi) {
    uint32_t amax = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = max(amax, __float_as_uint(fabsf(v[i])));
    const int s = mx_scale_exp(amax, 8);
    const float inv = mx_exp2i(-s);
    uint32_t w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        w[j] = mx_e4m3(v[4 * j] * inv) | (mx_e4m3(v[4 * j + 1] * inv) << 8) | (mx_e4m3(v[4 * j + 2] * inv) << 16) |
               (mx_e4m3(v[4 * j + 3] * inv) << 24);
    lo = make_uint4(w[0], w[1], w[2], w[3]);
    hi = make_uint4(w[4], w[5], w[6], w[7]);
    return static_cast<uint32_t>(s + 127);
}

__device__ __forceinline__ void bf16x32_to_float(const uint4 (&raw)[4], float (&v)[32]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t w[4] = {raw[q].x, raw[q].y, raw[q].z, raw[q].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[8 * q + 2 * j] = bf16lo(w[j]);
            v[8 * q + 2 * j + 1] = bf16hi(w[j]);
        }
    }
}

// Weight encoding: one thread per block of 32 values of one row.  rows and K
// multiples of 128.
template <bool W4>
__global__ void __launch_bounds__(256) mx_encode_weights_kernel(const __nv_bfloat16* __restrict__ w, long long rows,
                                                                int K, uint8_t* __restrict__ codes,
                                                                uint8_t* __restrict__ scales) {
    const int nb = K / 32;
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= rows * nb) return;
    const long long r = i / nb;
    const int b = static_cast<int>(i % nb);
    const uint4* src = reinterpret_cast<const uint4*>(w + r * K + b * 32);
    uint4 raw[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) raw[q] = src[q];
    float v[32];
    bf16x32_to_float(raw, v);
    uint32_t sbyte;
    if (W4) {
        uint32_t amax = 0;
#pragma unroll
        for (int k = 0; k < 32; ++k) amax = max(amax, __float_as_uint(fabsf(v[k])));
        const int s = mx_scale_exp(amax, 2);
        const float inv = mx_exp2i(-s);
        uint32_t wd[4] = {0, 0, 0, 0};
#pragma unroll
        for (int k = 0; k < 32; ++k) wd[k / 8] |= mx_e2m1(v[k] * inv) << (4 * (k % 8));
        *reinterpret_cast<uint4*>(codes + r * (K / 2) + b * 16) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        sbyte = static_cast<uint32_t>(s + 127);
    } else {
        uint4 lo, hi;
        sbyte = mx_encode32_e4m3(v, lo, hi);
        uint4* dst = reinterpret_cast<uint4*>(codes + r * K + b * 32);
        dst[0] = lo;
        dst[1] = hi;
    }
    const long long R = r / 128;
    const int m = static_cast<int>(r % 128), G = b / 4;
    scales[(R * (K / 128) + G) * 512 + (m % 32) * 16 + (m / 32) * 4 + (b % 4)] = static_cast<uint8_t>(sbyte);
}

// Decode regime: one warp per (token, slot) routed to an FFN expert.  The
// token's bf16 feature row is MXFP8-encoded into its sorted row.
static __global__ void __launch_bounds__(256) mx_gather_kernel(const int32_t* __restrict__ idx,
                                                               const int32_t* __restrict__ inv, int T, int K,
                                                               int n_ffn, const __nv_bfloat16* __restrict__ feat,
                                                               int ld_feat, int fdim, uint8_t* __restrict__ rows8,
                                                               int ld8, uint8_t* __restrict__ rows_sf, int ld_sf) {
    pdl_begin();
    const int lane = threadIdx.x & 31;
    const long i = static_cast<long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (i >= static_cast<long>(T) * K) return;
    const int e = idx[i];
    if (e < 0 || e >= n_ffn) return;
    const int t = static_cast<int>(i / K);
    const size_t row = static_cast<size_t>(inv[i]);
    for (int b = lane; b < fdim / 32; b += 32) {
        const uint4* src = reinterpret_cast<const uint4*>(feat + static_cast<size_t>(t) * ld_feat + b * 32);
        uint4 raw[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) raw[q] = src[q];
        float v[32];
        bf16x32_to_float(raw, v);
        uint4 lo, hi;
        const uint32_t sb = mx_encode32_e4m3(v, lo, hi);
        uint4* dst = reinterpret_cast<uint4*>(rows8 + row * ld8 + b * 32);
        dst[0] = lo;
        dst[1] = hi;
        rows_sf[row * ld_sf + (b >> 2) * 16 + (b & 3)] = static_cast<uint8_t>(sb);
    }
}

struct MxArgs {
    int K;                  // reduction length, multiple of 128
    int n_wtiles;           // 128-row weight tiles per expert
    const int4* list;       // {expert, first row, rows <= 32, 0}
    const int* count;       // entries in `list` (device)
    int w_rows_per_expert;  // rows of the weight tensor per expert (multiple of 128)
    int up_offset;          // gated: row offset of the up rows inside an expert (multiple of 128)
    const uint8_t* w_sf;    // weight scale atoms [rows/128][K/128][512]
    int n_out;              // valid output columns
    __nv_bfloat16* out;     // bf16 output (no re-encoding)
    int ld_out;
    uint8_t* out8;          // MXFP8 output codes [rows, ld_out8] and scales [rows, ld_out_sf] (16-byte chunks)
    uint8_t* out_sf;
    int ld_out8, ld_out_sf;
    int* err;
    unsigned long long timeout_ns;
};

template <int EPI, bool W4>
struct MxCfg {
    static constexpr int NT = 32;     // token rows per tile
    static constexpr int BK = 128;    // K elements per stage: 128 bytes per row in shared memory
    static constexpr int NA = (EPI == EPI_SWIGLU) ? 2 : 1;
    static constexpr int A_BYTES = 128 * BK;               // shared-memory bytes of a weight tile
    static constexpr int A_TX = W4 ? A_BYTES / 2 : A_BYTES; // bytes the copy reads (E2M1 arrives packed)
    static constexpr int B_BYTES = NT * BK;
    static constexpr int SF_BYTES = 512;
    static constexpr int OFF_B = NA * A_BYTES;
    static constexpr int OFF_SFA = OFF_B + B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + NA * SF_BYTES;
    static constexpr int STAGE_BYTES = (OFF_SFB + SF_BYTES + 1023) / 1024 * 1024;
    static constexpr int TX_BYTES = NA * A_TX + B_BYTES + (NA + 1) * SF_BYTES;
    static constexpr int STAGES = (NA == 2) ? 5 : 10;
    // Two accumulation chains per weight tile (even / odd K = 32 steps), so consecutive MMAs do not wait on
    // one another's accumulator; the epilogue adds them.  Chain c of weight tile a at column (c * NA + a) * NT.
    static constexpr int CHAINS = 2;
    static constexpr int ACC_COLS = CHAINS * NA * NT;  // one accumulator set (two sets: double buffering)
    // TMEM scale columns: a ring of SF_SLOTS slots after the accumulators; a slot holds the stage's weight
    // scales (4 columns per weight tile) and then its token scales (4 columns)
    static constexpr int SF_COL = 2 * ACC_COLS;
    static constexpr int SF_SLOT = 4 * (NA + 1);
    static constexpr int SF_SLOTS = 4;
    static constexpr int TMEM_COLS = SF_COL + SF_SLOTS * SF_SLOT <= 256 ? 256 : 512;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
    // every scale-factor address the MMA and tcgen05.cp see is a multiple of four columns
    static_assert(SF_COL % 4 == 0 && SF_COL + SF_SLOTS * SF_SLOT <= TMEM_COLS, "scale columns");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Weight-streaming GEMM with MX operands for experts that received <= 32 rows
// (D^T[128 x 32] = W_tile * X^T, the weight rows as the M = 128 operand).
// Per stage of 128 K elements: the weight tile(s) and the token tile by TMA
// (E2M1 weights through the packed-to-padded 16U4 copy), the weight scale
// atom(s) by a bulk copy, and the stage's 16-byte token-scale chunk of each
// token row by TMA.  The MMA thread moves each stage's scales into a ring of
// TMEM slots with tcgen05.cp and issues the stage's four K = 32 block-scaled
// MMAs, alternating between two accumulators.  With QOUT the epilogue applies the
// activation, stores it in bf16 precision and re-encodes it in MXFP8 (a warp
// holds one 32-column block of each token row).  Otherwise it writes bf16.
template <int EPI, bool W4, bool QOUT>
__global__ void __launch_bounds__(192, 1)
    tc_swap_mx_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                      const __grid_constant__ CUtensorMap tmXsf, const MxArgs args) {
    // The work list and the weights (codes and scales) are read before the wait for the previous kernel (see
    // pdl_wait); the token tiles, token scales and every output after it.
    using C = MxCfg<EPI, W4>;
    constexpr int NT = C::NT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* tfull = empty + C::STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = *args.count * args.n_wtiles;
    if (static_cast<int>(blockIdx.x) >= ntiles) {
        pdl_begin();
        return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmXsf);
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int nkb = args.K / C::BK;
    if (!(warp == 0 && lane == 0)) pdl_begin();

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            // The first STAGES stages' weight tiles and weight scales are requested before the wait for the
            // previous kernel (every slot is free then), their token tiles and token scales after it.
            uint32_t pre = 0;
            for (int t = blockIdx.x; t < ntiles && pre < C::STAGES; t += gridDim.x) {
                const int4 e = args.list[t / args.n_wtiles];
                const int wrow = e.x * args.w_rows_per_expert + (t % args.n_wtiles) * 128;
                const uint8_t* sfa0 = args.w_sf + static_cast<size_t>(wrow / 128) * nkb * C::SF_BYTES;
                const uint8_t* sfa1 = args.w_sf + static_cast<size_t>((wrow + args.up_offset) / 128) * nkb * C::SF_BYTES;
                for (int kb = 0; kb < nkb && pre < C::STAGES; ++kb, ++pre) {
                    uint8_t* st = smem + pre * C::STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[pre], C::TX_BYTES);
                    tma_load_2d(st, &tmW, &full[pre], kb * C::BK, wrow);
                    if (C::NA == 2) tma_load_2d(st + C::A_BYTES, &tmW, &full[pre], kb * C::BK, wrow + args.up_offset);
                    bulk_load(st + C::OFF_SFA, sfa0 + static_cast<size_t>(kb) * C::SF_BYTES, C::SF_BYTES, &full[pre]);
                    if (C::NA == 2)
                        bulk_load(st + C::OFF_SFA + C::SF_BYTES, sfa1 + static_cast<size_t>(kb) * C::SF_BYTES,
                                  C::SF_BYTES, &full[pre]);
                }
            }
            pdl_begin();
            uint32_t kc = 0;
            uint32_t last_parity[C::STAGES];
            bool issued[C::STAGES];
            for (int s = 0; s < C::STAGES; ++s) issued[s] = false, last_parity[s] = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                const int4 e = args.list[t / args.n_wtiles];
                const int wrow = e.x * args.w_rows_per_expert + (t % args.n_wtiles) * 128;
                const uint8_t* sfa0 = args.w_sf + static_cast<size_t>(wrow / 128) * nkb * C::SF_BYTES;
                const uint8_t* sfa1 = args.w_sf + static_cast<size_t>((wrow + args.up_offset) / 128) * nkb * C::SF_BYTES;
                for (int kb = 0; kb < nkb; ++kb, ++kc) {
                    const int s = kc % C::STAGES;
                    const uint32_t ph = (kc / C::STAGES) & 1;
                    uint8_t* st = smem + s * C::STAGE_BYTES;
                    if (kc >= pre) {
                        if (!mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag, args.err, args.timeout_ns)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&full[s], C::TX_BYTES);
                        tma_load_2d(st, &tmW, &full[s], kb * C::BK, wrow);
                        if (C::NA == 2)
                            tma_load_2d(st + C::A_BYTES, &tmW, &full[s], kb * C::BK, wrow + args.up_offset);
                        bulk_load(st + C::OFF_SFA, sfa0 + static_cast<size_t>(kb) * C::SF_BYTES, C::SF_BYTES,
                                  &full[s]);
                        if (C::NA == 2)
                            bulk_load(st + C::OFF_SFA + C::SF_BYTES, sfa1 + static_cast<size_t>(kb) * C::SF_BYTES,
                                      C::SF_BYTES, &full[s]);
                    }
                    tma_load_2d(st + C::OFF_B, &tmX, &full[s], kb * C::BK, e.y);
                    tma_load_2d(st + C::OFF_SFB, &tmXsf, &full[s], kb * 16, e.y);
                    issued[s] = true;
                    last_parity[s] = ph;
                }
            }
            for (int s = 0; s < C::STAGES; ++s)
                if (issued[s]) {
                    int no_abort = 0;
                    const uint64_t drain = args.timeout_ns > 200000000ull ? args.timeout_ns : 200000000ull;
                    mbar_wait_bounded(&full[s], last_parity[s], &no_abort, args.err, drain);
                }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            constexpr uint32_t idesc = umma_idesc_mx(128, NT, W4 ? MXF_E2M1 : MXF_E4M3, MXF_E4M3);
            uint32_t kc = 0;
            int it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++it) {
                const int buf = it & 1;
                const uint32_t use = (it >> 1) & 1;
                if (!mbar_wait_bounded(&tempty[buf], use ^ 1, abort_flag, args.err, args.timeout_ns)) break;
                tc_fence_after();
                const uint32_t d0 = tmem_base + buf * C::ACC_COLS;
                for (int kb = 0; kb < nkb; ++kb, ++kc) {
                    const int s = kc % C::STAGES;
                    const uint32_t ph = (kc / C::STAGES) & 1;
                    if (!mbar_wait_bounded(&full[s], ph, abort_flag, args.err, args.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + s * C::STAGE_BYTES);
                    const uint32_t sf_a0 = tmem_base + C::SF_COL + (kc % C::SF_SLOTS) * C::SF_SLOT;
                    const uint32_t sf_a1 = sf_a0 + 4, sf_b = sf_a0 + 4 * C::NA;
                    tmem_cp_32x128b_x4(sf_a0, umma_desc_plain(st + C::OFF_SFA, 128));
                    if (C::NA == 2) tmem_cp_32x128b_x4(sf_a1, umma_desc_plain(st + C::OFF_SFA + C::SF_BYTES, 128));
                    tmem_cp_32x128b_x4(sf_b, umma_desc_plain(st + C::OFF_SFB, 128));
                    const uint64_t a0 = umma_desc_sw128(st);
                    const uint64_t a1 = umma_desc_sw128(st + C::A_BYTES);
                    const uint64_t bx = umma_desc_sw128(st + C::OFF_B);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t c = kk & 1;                                 // accumulation chain
                        const uint32_t acc = (kb > 0 || kk >= C::CHAINS) ? 1u : 0u;  // first step of a chain: overwrite
                        const uint32_t id = idesc | umma_idesc_sf_ids(kk, kk);
                        umma_mx(d0 + c * C::NA * NT, a0 + 2 * kk, bx + 2 * kk, id, sf_a0, sf_b, acc);
                        if (C::NA == 2) umma_mx(d0 + (c * C::NA + 1) * NT, a1 + 2 * kk, bx + 2 * kk, id, sf_a1, sf_b, acc);
                    }
                    umma_commit(&empty[s]);
                }
                if (ok) umma_commit(&tfull[buf]);
            }
            umma_commit(mma_done);
            int no_abort = 0;
            const uint64_t drain = args.timeout_ns > 200000000ull ? args.timeout_ns : 200000000ull;
            mbar_wait_bounded(mma_done, 0, &no_abort, args.err, drain);
        }
    } else {
        // ---------------------------------------------------- epilogue: thread = output column
        const int quad = warp & 3;
        int it = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
            const int4 e = args.list[t / args.n_wtiles];
            const int col = (t % args.n_wtiles) * 128 + quad * 32 + lane;
            const int buf = it & 1;
            const uint32_t use = (it >> 1) & 1;
            int ok = 1;
            if (lane == 0) ok = mbar_wait_bounded(&tfull[buf], use, abort_flag, args.err, args.timeout_ns) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + buf * C::ACC_COLS + (static_cast<uint32_t>(quad * 32) << 16);
            const bool valid = col < args.n_out;
            uint8_t* dst8 = QOUT ? args.out8 + static_cast<size_t>(e.y) * args.ld_out8 + col : nullptr;
            uint8_t* sdst = QOUT ? args.out_sf + static_cast<size_t>(e.y) * args.ld_out_sf + (col >> 7) * 16 + ((col >> 5) & 3)
                                 : nullptr;
            __nv_bfloat16* dst = QOUT ? nullptr : args.out + static_cast<size_t>(e.y) * args.ld_out + col;
            // Only the expert's rows in this tile (e.z, the same for the whole warp), one at a time, each row's
            // accumulator columns (the two chains) read from tensor memory and added.  A small loop keeps the
            // epilogue's code small, so the other warps do not stall on instruction fetch.
            for (int j = 0; j < e.z; ++j) {
                uint32_t c0, c1, c2 = 0u, c3 = 0u;
                tmem_ld_32x32b_x1(taddr + j, c0);
                tmem_ld_32x32b_x1(taddr + C::NA * NT + j, c1);
                if (C::NA == 2) {
                    tmem_ld_32x32b_x1(taddr + NT + j, c2);
                    tmem_ld_32x32b_x1(taddr + 3 * NT + j, c3);
                }
                tmem_ld_wait();
                float a = __uint_as_float(c0) + __uint_as_float(c1);
                if (EPI == EPI_RELU2) a = act_relu2(a);
                if (EPI == EPI_SWIGLU) a = act_silu_mul(a, __uint_as_float(c2) + __uint_as_float(c3));
                if (QOUT) {
                    // the stored (bf16) activation, its block maximum over the warp (the warp's 32 columns are
                    // one block), the E8M0 scale, the E4M3 codes; lane 0 writes the block scale
                    const float v = valid ? __bfloat162float(__float2bfloat16_rn(a)) : 0.f;
                    const int sx = mx_scale_exp(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(v))), 8);
                    if (valid) dst8[static_cast<size_t>(j) * args.ld_out8] = static_cast<uint8_t>(mx_e4m3(v * mx_exp2i(-sx)));
                    if (lane == 0) sdst[static_cast<size_t>(j) * args.ld_out_sf] = static_cast<uint8_t>(sx + 127);
                } else if (valid) {
                    dst[static_cast<size_t>(j) * args.ld_out] = __float2bfloat16_rn(a);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[buf]);  // this tile's accumulator is free for the MMA warp
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace lmoe
