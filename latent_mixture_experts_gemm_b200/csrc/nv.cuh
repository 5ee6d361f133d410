// nv.cuh -- NVFP4 expert weights: encoding, the token-operand encoding, and the
// decode-regime weight-streaming GEMM on tcgen05 kind::mxf4nvf4 MMAs.
//
// Format (NVIDIA's two-level NVFP4; the pages name it as Nemotron 3 Super's
// training format, in the training note of the outlook section): E2M1
// elements; a block of 16 consecutive values along K shares one positive E4M3
// scale sb; a tensor shares one fp32 scale g.  A weight matrix (one expert's
// W1_e or W2_e) takes g = amax / (6 * 448), or 1 when all zero; the token
// operands take g = 1.  sb = E4M3(amax_block / (g * 6)) and each element is
// E2M1(v / (sb * g)), both rounded to nearest even and saturated (448, 6); a
// block whose scale is zero encodes zeros.  The products g * 6 and sb * g and
// both quotients are fp32 operations, rounded to nearest.
//
// Both MMA operands are NVFP4 (the block-16 MMA kind takes E2M1 on both
// sides).  The MMA applies both operands' block scales; the epilogue applies
// the weight matrix's g.
//
// Weight layout in HBM:
//   codes   [rows, K/2] bytes, element 2i in the low nibble of byte i
//   scales  E4M3 bytes in 512-byte atoms [rows/128][K/64][32][16]: byte
//           (r, c) of atom (R, G) is the scale of row 128R + 32(c/4) + r,
//           block 4G + (c % 4) (block = 16 elements): the order the tensor
//           cores read block scales in, one atom per MMA (K = 64)
//   gscale  fp32 [matrices]
// Token-operand layout (workspace): codes [rows, K/2] bytes; scales planar
// [K/64][rows][16] bytes: chunk c of row r holds, in its first four bytes, the
// scales of the row's elements 64c .. 64c+63 (the other twelve are not read).
// Seen as 8-byte elements [K/64][2 * rows], one copy of 4 chunks x 64 elements
// (four 512-byte rows) lands as the four 512-byte atoms of one 256-element
// stage (the first 32 rows of each 128-row atom).
#pragma once
#include "mx.cuh"

namespace lmoe {

// Value of an E4M3 code (exact in fp32).
__device__ __forceinline__ float nv_e4m3_value(uint32_t code) {
    const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code), __NV_E4M3);
    return __half2float(__half(h));
}

// Encode 16 bf16-exact values with tensor scale g: the packed codes (element 2i in the low nibble of byte i)
// and the E4M3 scale byte.
__device__ __forceinline__ uint32_t nv_encode16(const float (&v)[16], float g, uint2& packed) {
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const uint32_t sb = mx_e4m3(__fdiv_rn(amax, __fmul_rn(g, 6.0f)));
    const float sg = __fmul_rn(nv_e4m3_value(sb), g);
    uint32_t w[2] = {0u, 0u};
    if (sb != 0) {
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i / 8] |= mx_e2m1(__fdiv_rn(v[i], sg)) << (4 * (i % 8));
    }
    packed = make_uint2(w[0], w[1]);
    return sb;
}

// E2M1 code (sign in bit 3) of v / s for v exact in bf16 and s an E4M3 value, without the division: |v| is
// compared with the seven midpoints between the E2M1 magnitudes times s (products exact in fp32), a tie going
// to the even code; past 6 it saturates.  The codes equal those of rounding the fp32 quotient v / s: that
// quotient can equal a midpoint only when v is exactly the midpoint times s (v has 8 significant bits and the
// products at most 7, so they differ by far more than the quotient's rounding otherwise).
__device__ __forceinline__ uint32_t nv_e2m1_code(float v, float s) {
    const float a = fabsf(v);
    const uint32_t m = (a > 0.25f * s) + (a >= 0.75f * s) + (a > 1.25f * s) + (a >= 1.75f * s) + (a > 2.5f * s) +
                       (a >= 3.5f * s) + (a > 5.0f * s);
    return m | ((__float_as_uint(v) >> 28) & 8u);
}

__device__ __forceinline__ void bf16x16_to_float(const uint4 (&raw)[2], float (&v)[16]) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const uint32_t w[4] = {raw[q].x, raw[q].y, raw[q].z, raw[q].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[8 * q + 2 * j] = bf16lo(w[j]);
            v[8 * q + 2 * j + 1] = bf16hi(w[j]);
        }
    }
}

// Largest |w| of each matrix of n_per_mat values (blockIdx.y = matrix), as the bit pattern of a non-negative
// float: the unsigned maximum of those patterns is the pattern of the maximum.  gbits zeroed before.
__global__ void __launch_bounds__(256) nv_amax_kernel(const __nv_bfloat16* __restrict__ w, long long n_per_mat,
                                                      uint32_t* __restrict__ gbits) {
    const int mat = blockIdx.y;
    const uint4* src = reinterpret_cast<const uint4*>(w + static_cast<size_t>(mat) * n_per_mat);
    const long long n8 = n_per_mat / 8;
    uint32_t m = 0;
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const uint4 q = src[i];
        const uint32_t wd[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            m = max(m, __float_as_uint(fabsf(bf16lo(wd[j]))));
            m = max(m, __float_as_uint(fabsf(bf16hi(wd[j]))));
        }
    }
    m = __reduce_max_sync(0xffffffffu, m);
    if ((threadIdx.x & 31) == 0 && m != 0) atomicMax(&gbits[mat], m);
}

// g = amax / (6 * 448) in place of the amax bits (1 for an all-zero matrix).
__global__ void nv_tensor_scale_kernel(uint32_t* __restrict__ gbits, int n_mats) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n_mats) return;
    const uint32_t b = gbits[i];
    const float g = b == 0 ? 1.0f : __fdiv_rn(__uint_as_float(b), 2688.0f);
    gbits[i] = __float_as_uint(g);
}

// Weight encoding: one thread per block of 16 values of one row; row r belongs to matrix r / rows_per_mat.
// rows_per_mat a multiple of 128, K of 64.
__global__ void __launch_bounds__(256) nv_encode_weights_kernel(const __nv_bfloat16* __restrict__ w, long long rows,
                                                                long long rows_per_mat, int K,
                                                                const float* __restrict__ g,
                                                                uint8_t* __restrict__ codes,
                                                                uint8_t* __restrict__ scales) {
    const int nb = K / 16;
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= rows * nb) return;
    const long long r = i / nb;
    const int b = static_cast<int>(i % nb);
    const uint4* src = reinterpret_cast<const uint4*>(w + r * K + b * 16);
    uint4 raw[2] = {src[0], src[1]};
    float v[16];
    bf16x16_to_float(raw, v);
    uint2 p;
    const uint32_t sb = nv_encode16(v, g[r / rows_per_mat], p);
    *reinterpret_cast<uint2*>(codes + r * (K / 2) + b * 8) = p;
    const long long R = r / 128;
    const int m = static_cast<int>(r % 128), G = b / 4;
    scales[(R * (K / 64) + G) * 512 + (m % 32) * 16 + (m / 32) * 4 + (b % 4)] = static_cast<uint8_t>(sb);
}

// Decode regime: one warp per (token, slot) routed to an FFN expert.  The token's bf16 feature row is
// NVFP4-encoded (g = 1) into its sorted row: codes [rows, fdim/2], scale chunks planar [fdim/64][sf_rows][16].
static __global__ void __launch_bounds__(256) nv_gather_kernel(const int32_t* __restrict__ idx,
                                                               const int32_t* __restrict__ inv, int T, int K,
                                                               int n_ffn, const __nv_bfloat16* __restrict__ feat,
                                                               int ld_feat, int fdim, uint8_t* __restrict__ rows4,
                                                               uint8_t* __restrict__ rows_sf, int sf_rows) {
    pdl_begin();
    const int lane = threadIdx.x & 31;
    const long i = static_cast<long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (i >= static_cast<long>(T) * K) return;
    const int e = idx[i];
    if (e < 0 || e >= n_ffn) return;
    const int t = static_cast<int>(i / K);
    const size_t row = static_cast<size_t>(inv[i]);
    for (int b = lane; b < fdim / 16; b += 32) {
        const uint4* src = reinterpret_cast<const uint4*>(feat + static_cast<size_t>(t) * ld_feat + b * 16);
        uint4 raw[2] = {src[0], src[1]};
        float v[16];
        bf16x16_to_float(raw, v);
        uint2 p;
        const uint32_t sb = nv_encode16(v, 1.0f, p);
        *reinterpret_cast<uint2*>(rows4 + row * (fdim / 2) + b * 8) = p;
        rows_sf[(static_cast<size_t>(b / 4) * sf_rows + row) * 16 + (b % 4)] = static_cast<uint8_t>(sb);
    }
}

struct NvArgs {
    int K;                  // reduction length, multiple of 256
    int n_wtiles;           // 128-row weight tiles per expert
    const int4* list;       // {expert, first row, rows <= 32, 0}
    const int* count;       // entries in `list` (device)
    int w_rows_per_expert;  // rows of the weight tensor per expert (multiple of 128)
    int up_offset;          // gated: row offset of the up rows inside an expert (multiple of 128)
    const uint8_t* w_sf;    // weight scale atoms [rows/128][K/64][512]
    const float* w_g;       // fp32 tensor scale of each expert's matrix
    int n_out;              // valid output columns
    __nv_bfloat16* out;     // bf16 output (no re-encoding)
    int ld_out;
    uint8_t* out4;          // NVFP4 output codes [rows, n_out/2] and planar scale chunks [n_out/64][sf_rows][16]
    uint8_t* out_sf;
    int sf_rows;
    int* err;
    unsigned long long timeout_ns;
};

template <int EPI>
struct NvCfg {
    static constexpr int NT = 32;       // token rows per tile
    static constexpr int BK = 256;      // K elements per stage: 128 packed bytes per row in shared memory
    static constexpr int MMAS = BK / 64;
    static constexpr int NA = (EPI == EPI_SWIGLU) ? 2 : 1;
    static constexpr int A_BYTES = 128 * BK / 2;
    static constexpr int B_BYTES = NT * BK / 2;
    static constexpr int ATOM = 512;    // the scales of one MMA for 128 rows
    static constexpr int OFF_B = NA * A_BYTES;
    static constexpr int OFF_SFA = OFF_B + B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + NA * MMAS * ATOM;
    static constexpr int STAGE_BYTES = (OFF_SFB + MMAS * ATOM + 1023) / 1024 * 1024;
    static constexpr int TX_BYTES = NA * A_BYTES + B_BYTES + (NA + 1) * MMAS * ATOM;
    static constexpr int STAGES = (NA == 2) ? 5 : 9;
    // two accumulation chains per weight tile (even / odd MMAs), added by the epilogue; chain c of weight
    // tile a at column (c * NA + a) * NT
    static constexpr int CHAINS = 2;
    static constexpr int ACC_COLS = CHAINS * NA * NT;
    // TMEM scale columns: one slot per shared-memory stage after the two accumulator sets; a slot holds a
    // stage's scales, 4 columns per MMA: weight tile 0's MMAs, then tile 1's (gated), then the token rows'
    // (the order of the atoms in the stage's shared memory)
    static constexpr int SF_COL = 2 * ACC_COLS;
    static constexpr int SF_SLOT = 4 * MMAS * (NA + 1);
    static constexpr int SF_SLOTS = STAGES;
    static constexpr int TMEM_COLS = SF_COL + SF_SLOTS * SF_SLOT <= 256 ? 256 : 512;
    // warps: 0 TMA, 1 MMA, 2-5 epilogue, 6-9 scales (one per TMEM lane quadrant)
    static constexpr int THREADS = 320;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 512;
    static_assert(SF_COL % 4 == 0 && SF_SLOT % 4 == 0 && SF_COL + SF_SLOTS * SF_SLOT <= TMEM_COLS, "scale columns");
    static_assert(STAGE_BYTES % 1024 == 0 && SMEM_BYTES <= 232448, "shared memory");
    static_assert(MMAS == 4, "the scale warps store four atoms (16 columns) at a time");
};

// Weight-streaming GEMM with NVFP4 operands for experts that received <= 32
// rows (D^T[128 x 32] = W_tile * X^T, the weight rows as the M = 128 operand).
// Per stage of 256 K elements: the weight tile(s) and the token tile by TMA,
// the weight scale atoms (one per MMA) by a bulk copy, and the token scale
// atoms by one TMA copy of four 512-byte rows.  Four scale warps, one per TMEM
// lane quadrant, store each stage's atoms into the stage's TMEM slot
// (tcgen05.st, outside the tensor-core pipe: eight tcgen05.cp per stage in
// that pipe measured 12 us slower per launch); the MMA thread issues four
// K = 64 MMAs, alternating between two accumulators.  The epilogue multiplies
// by the expert matrix's g; with QOUT it applies the activation, stores it in
// bf16 precision and re-encodes it in NVFP4 (g = 1): a 16-column block of a
// token row is held by 16 lanes of a warp.  Otherwise it writes bf16.
template <int EPI, bool QOUT>
__global__ void __launch_bounds__(NvCfg<EPI>::THREADS, 1)
    tc_swap_nv_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                      const __grid_constant__ CUtensorMap tmXsf, const NvArgs args) {
    // The work list and the weights (codes and scales) are read before the wait for the previous kernel (see
    // pdl_wait); the token tiles, token scales and every output after it.
    using C = NvCfg<EPI>;
    constexpr int NT = C::NT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* tfull = empty + C::STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint64_t* sfull = mma_done + 1;  // a stage's scales are in its TMEM slot (one arrival per scale warp)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sfull + C::STAGES);
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
            mbar_init(&sfull[s], 4);
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
    constexpr int STAGE_SF = C::MMAS * C::ATOM;  // weight scale bytes of one stage and weight tile
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
                const uint8_t* sfa0 = args.w_sf + static_cast<size_t>(wrow / 128) * (args.K / 64) * C::ATOM;
                const uint8_t* sfa1 =
                    args.w_sf + static_cast<size_t>((wrow + args.up_offset) / 128) * (args.K / 64) * C::ATOM;
                for (int kb = 0; kb < nkb && pre < C::STAGES; ++kb, ++pre) {
                    uint8_t* st = smem + pre * C::STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[pre], C::TX_BYTES);
                    tma_load_2d(st, &tmW, &full[pre], kb * (C::BK / 2), wrow);
                    if (C::NA == 2)
                        tma_load_2d(st + C::A_BYTES, &tmW, &full[pre], kb * (C::BK / 2), wrow + args.up_offset);
                    bulk_load(st + C::OFF_SFA, sfa0 + static_cast<size_t>(kb) * STAGE_SF, STAGE_SF, &full[pre]);
                    if (C::NA == 2)
                        bulk_load(st + C::OFF_SFA + STAGE_SF, sfa1 + static_cast<size_t>(kb) * STAGE_SF, STAGE_SF,
                                  &full[pre]);
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
                const uint8_t* sfa0 = args.w_sf + static_cast<size_t>(wrow / 128) * (args.K / 64) * C::ATOM;
                const uint8_t* sfa1 =
                    args.w_sf + static_cast<size_t>((wrow + args.up_offset) / 128) * (args.K / 64) * C::ATOM;
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
                        tma_load_2d(st, &tmW, &full[s], kb * (C::BK / 2), wrow);
                        if (C::NA == 2)
                            tma_load_2d(st + C::A_BYTES, &tmW, &full[s], kb * (C::BK / 2), wrow + args.up_offset);
                        bulk_load(st + C::OFF_SFA, sfa0 + static_cast<size_t>(kb) * STAGE_SF, STAGE_SF, &full[s]);
                        if (C::NA == 2)
                            bulk_load(st + C::OFF_SFA + STAGE_SF, sfa1 + static_cast<size_t>(kb) * STAGE_SF,
                                      STAGE_SF, &full[s]);
                    }
                    tma_load_2d(st + C::OFF_B, &tmX, &full[s], kb * (C::BK / 2), e.y);
                    tma_load_2d(st + C::OFF_SFB, &tmXsf, &full[s], 2 * e.y, kb * C::MMAS);
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
            constexpr uint32_t idesc = umma_idesc_nvf4(128, NT);
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
                    if (!mbar_wait_bounded(&sfull[s], ph, abort_flag, args.err, args.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + s * C::STAGE_BYTES);
                    const uint32_t slot = tmem_base + C::SF_COL + s * C::SF_SLOT;
                    const uint32_t sf_a1 = slot + 4 * C::MMAS, sf_b = slot + 4 * C::MMAS * C::NA;
                    const uint64_t a0 = umma_desc_sw128(st);
                    const uint64_t a1 = umma_desc_sw128(st + C::A_BYTES);
                    const uint64_t bx = umma_desc_sw128(st + C::OFF_B);
#pragma unroll
                    for (int kk = 0; kk < C::MMAS; ++kk) {
                        const uint32_t c = kk & 1;                                   // accumulation chain
                        const uint32_t acc = (kb > 0 || kk >= C::CHAINS) ? 1u : 0u;  // first step of a chain: overwrite
                        umma_nv(d0 + c * C::NA * NT, a0 + 2 * kk, bx + 2 * kk, idesc, slot + 4 * kk, sf_b + 4 * kk, acc);
                        if (C::NA == 2)
                            umma_nv(d0 + (c * C::NA + 1) * NT, a1 + 2 * kk, bx + 2 * kk, idesc, sf_a1 + 4 * kk,
                                    sf_b + 4 * kk, acc);
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
    } else if (warp >= 6) {
        // ---------------------------------------------------- scale warps
        // The stage's (NA + 1) * MMAS atoms lie in shared memory in the order of the slot's columns (weight
        // tile 0's, tile 1's, the token rows'), 4 columns each: each lane stores its row of every atom, in
        // its warp's lane quadrant, four atoms per store.
        const uint32_t quadrant = static_cast<uint32_t>((warp & 3) * 32) << 16;
        uint32_t kc = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            for (int kb = 0; kb < nkb; ++kb, ++kc) {
                const int s = kc % C::STAGES;
                const uint32_t ph = (kc / C::STAGES) & 1;
                // every lane observes the copy's completion before it reads the stage's shared memory
                const bool got = mbar_wait_bounded(&full[s], ph, abort_flag, args.err, args.timeout_ns);
                if (!__all_sync(0xffffffffu, got)) {
                    ok = false;
                    break;
                }
                const uint8_t* atoms = smem + s * C::STAGE_BYTES + C::OFF_SFA;
                const uint32_t taddr = tmem_base + quadrant + C::SF_COL + s * C::SF_SLOT;
#pragma unroll
                for (int g = 0; g < C::NA + 1; ++g) {
                    uint32_t r[16];
#pragma unroll
                    for (int kk = 0; kk < C::MMAS; ++kk) atom_row(atoms + (g * C::MMAS + kk) * C::ATOM, lane, r + 4 * kk);
                    tmem_st_32x32b_x16(taddr + 16 * g, r);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sfull[s]);
            }
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
            const float gw = args.w_g[e.x];
            const bool valid = col < args.n_out;
            const uint32_t half = lane < 16 ? 0x0000ffffu : 0xffff0000u;
            uint8_t* dst4 = QOUT ? args.out4 + static_cast<size_t>(e.y) * (args.n_out / 2) + (col >> 1) : nullptr;
            uint8_t* sdst = QOUT ? args.out_sf + (static_cast<size_t>(col >> 6) * args.sf_rows + e.y) * 16 + ((col >> 4) & 3)
                                 : nullptr;
            __nv_bfloat16* dst = QOUT ? nullptr : args.out + static_cast<size_t>(e.y) * args.ld_out + col;
            // Only the expert's rows in this tile (e.z, the same for the whole warp: one or two at decode), one
            // at a time, each row's accumulator columns read from tensor memory: the two chains are added and
            // scaled by the weight matrix's g.  A small loop, so the epilogue's code stays small (an unrolled
            // one over all 32 rows stalled the other warps on instruction fetch).
            for (int j = 0; j < e.z; ++j) {
                uint32_t c0, c1, c2 = 0u, c3 = 0u;
                tmem_ld_32x32b_x1(taddr + j, c0);
                tmem_ld_32x32b_x1(taddr + C::NA * NT + j, c1);
                if (C::NA == 2) {
                    tmem_ld_32x32b_x1(taddr + NT + j, c2);
                    tmem_ld_32x32b_x1(taddr + 3 * NT + j, c3);
                }
                tmem_ld_wait();
                float a = (__uint_as_float(c0) + __uint_as_float(c1)) * gw;
                if (EPI == EPI_RELU2) a = act_relu2(a);
                if (EPI == EPI_SWIGLU) a = act_silu_mul(a, (__uint_as_float(c2) + __uint_as_float(c3)) * gw);
                if (QOUT) {
                    // the stored (bf16) activation; the block maximum over the 16 lanes that hold the block
                    // (lanes 0-15 and 16-31, one reduction per half); the E4M3 scale; the codes (nv_e2m1_code:
                    // the same codes as dividing by the scale); lane pairs form bytes, lanes 0, 8, 16, 24 store
                    // 4-byte words and lanes 0 and 16 the block scales
                    const float v = valid ? __bfloat162float(__float2bfloat16_rn(a)) : 0.f;
                    const uint32_t amax = __reduce_max_sync(half, __float_as_uint(fabsf(v)));
                    const uint32_t sb = mx_e4m3(__fdiv_rn(__uint_as_float(amax), 6.0f));
                    uint32_t w = sb != 0 ? nv_e2m1_code(v, nv_e4m3_value(sb)) : 0u;
                    w |= __shfl_down_sync(0xffffffffu, w, 1) << 4;
                    w |= (__shfl_down_sync(0xffffffffu, w, 2) << 8) | (__shfl_down_sync(0xffffffffu, w, 4) << 16) |
                         (__shfl_down_sync(0xffffffffu, w, 6) << 24);
                    if (valid) {
                        if ((lane & 7) == 0)
                            *reinterpret_cast<uint32_t*>(dst4 + static_cast<size_t>(j) * (args.n_out / 2)) = w;
                        if ((lane & 15) == 0) sdst[static_cast<size_t>(j) * 16] = static_cast<uint8_t>(sb);
                    }
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
