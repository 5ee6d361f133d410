// tc_swap.cuh -- tcgen05 weight-streaming GEMM for experts that received few rows.
//
// In the decode regime an expert sees ~1-16 rows, so its cost is reading its
// weights once.  The GEMM is therefore computed transposed ("swap-AB"): the
// expert's weight rows are the M = 128 operand and its token rows the N = NT
// operand, D^T[128 x NT] = W_tile[128 x K] * X[NT x K]^T.  TMA streams 16 KB
// weight tiles through a deep shared-memory ring; one thread issues the MMAs;
// four epilogue warps read D^T back (thread = output column, registers = token
// rows) and write the rows of the expert's output.  Nothing but the TMA issue
// and the epilogue runs on the SM's CUDA cores, so the kernel streams at HBM
// speed.
//
// Tiles: one work-list entry (expert, first row, rows <= NT) times the
// expert's 128-row weight tiles; gated experts load the gate tile and the
// matching up tile into two accumulators so one thread sees both.
//
// Dense mode (no list: one entry covering the first `dense_rows` rows) serves
// the few-token projections: the weight rows of `tmW` come first, those of
// `tmW2` after them, and K may be split `k_splits` ways so that more CTAs
// stream the weights (the host takes 512-deep slices, 128 KB of weights per
// (tile, split) unit, at most one unit per SM).  With `partial` set, each
// (tile, split) writes its fp32 partial sums to partial[split][weight row][NT];
// swap_reduce_kernel then adds the splits in order (deterministic) and applies
// the epilogue.
#pragma once
#include "tc_gemm.cuh"

namespace lmoe {

struct SwapArgs {
    int K;                  // reduction length, multiple of 64
    int n_wtiles;           // 128-row weight tiles per expert (dense mode: of both weight maps)
    int n_wtiles0;          // dense mode: tiles that come from tmW (the rest from tmW2)
    int k_splits;           // K split this many ways (values below 1 mean 1)
    const int4* list;       // {expert, first row, rows, 0}; nullptr => dense mode
    const int* count;       // entries in `list` (device)
    int dense_rows;         // dense mode: token rows (<= NT)
    float* partial;         // non-null: write fp32 partials [k_splits][part_rows][NT] instead of `out`
    int part_rows;          // rows of one split in `partial`
    int w_rows_per_expert;  // rows of the weight tensor per expert
    int up_offset;          // gated: row offset of the up rows inside an expert
    int n_out;              // valid output columns
    __nv_bfloat16* out;
    int ld_out;
    int* err;
    unsigned long long timeout_ns;
    // Two-part token operand (dense mode): with k_wrap > 0, K = 2 * k_wrap and k-blocks at or past k_wrap
    // read their token tile from tmX2 and their weight tile at k - k_wrap: W * (X + X2)^T, the weights
    // streamed twice.
    int k_wrap;
};

template <int NT, int EPI>
struct SwapCfg {
    static constexpr int BK = 64;
    static constexpr int NA = (EPI == EPI_SWIGLU) ? 2 : 1;  // weight tiles per stage
    static constexpr int A_BYTES = 128 * BK * 2;
    static constexpr int B_BYTES = NT * BK * 2;
    static constexpr int STAGE_BYTES = NA * A_BYTES + B_BYTES;
    static constexpr int STAGES = (NA == 2) ? 6 : 10;
    static constexpr int ACC_COLS = NA * NT;  // columns of one accumulator set
    static constexpr int TMEM_COLS = (2 * ACC_COLS <= 32) ? 32 : (2 * ACC_COLS <= 64 ? 64 : 128);
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
    static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte swizzle-atom alignment");
};

template <int NT>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[NT]);
template <>
__device__ __forceinline__ void tmem_ld_cols<16>(uint32_t taddr, uint32_t (&r)[16]) {
    tmem_ld_32x32b_x16(taddr, r);
}
template <>
__device__ __forceinline__ void tmem_ld_cols<32>(uint32_t taddr, uint32_t (&r)[32]) {
    tmem_ld_32x32b_x32(taddr, r);
}

struct SwapJob {
    int4 e;      // {expert, first row, rows}
    int wt;      // weight tile
    int split;   // K split
    int kb0, kb1;
    int wrow;    // first weight row in its tensor map
    bool second; // dense mode: the tile comes from tmW2
};

__device__ __forceinline__ int swap_splits(const SwapArgs& a) { return a.k_splits > 1 ? a.k_splits : 1; }

__device__ __forceinline__ int swap_total(const SwapArgs& a) {
    const int entries = a.list != nullptr ? *a.count : 1;
    return entries * a.n_wtiles * swap_splits(a);
}

__device__ __forceinline__ void swap_job(const SwapArgs& a, int t, int nkb, SwapJob& j) {
    const int S = swap_splits(a);
    const int per_entry = a.n_wtiles * S;
    const int entry = t / per_entry, rem = t % per_entry;
    j.wt = rem / S;
    j.split = rem % S;
    j.kb0 = (j.split * nkb) / S;
    j.kb1 = ((j.split + 1) * nkb) / S;
    if (a.list != nullptr) {
        j.e = a.list[entry];
        j.second = false;
        j.wrow = j.e.x * a.w_rows_per_expert + j.wt * 128;
    } else {
        j.e = make_int4(0, 0, a.dense_rows, 0);
        j.second = j.wt >= a.n_wtiles0;
        j.wrow = (j.second ? j.wt - a.n_wtiles0 : j.wt) * 128;
    }
}

template <int NT, int EPI>
__global__ void __launch_bounds__(192, 1)
    tc_swap_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                   const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmX2,
                   const SwapArgs args) {
    // No pdl_begin() here: the work list (from the dispatch, two or more launches back) and the weights are
    // read before the wait for the previous kernel; the token tiles and every output after it.
    using C = SwapCfg<NT, EPI>;
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
    const int ntiles = swap_total(args);
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
        if (args.list == nullptr) tma_prefetch_desc(&tmW2);
        if (args.k_wrap > 0) tma_prefetch_desc(&tmX2);
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
            // The first STAGES stages' weight tiles are requested before the wait for the previous kernel
            // (every slot is free then), their token tiles after it; each stage's barrier expects both.
            uint32_t pre = 0;
            for (int t = blockIdx.x; t < ntiles && pre < C::STAGES; t += gridDim.x) {
                SwapJob j;
                swap_job(args, t, nkb, j);
                const CUtensorMap* wmap = j.second ? &tmW2 : &tmW;
                for (int kb = j.kb0; kb < j.kb1 && pre < C::STAGES; ++kb, ++pre) {
                    uint8_t* st = smem + pre * C::STAGE_BYTES;
                    const bool x2 = args.k_wrap > 0 && kb * C::BK >= args.k_wrap;
                    const int kx = x2 ? kb * C::BK - args.k_wrap : kb * C::BK;
                    mbar_arrive_expect_tx(&full[pre], C::STAGE_BYTES);
                    tma_load_2d(st, wmap, &full[pre], kx, j.wrow);
                    if (C::NA == 2) tma_load_2d(st + C::A_BYTES, wmap, &full[pre], kx, j.wrow + args.up_offset);
                }
            }
            pdl_begin();
            uint32_t kc = 0;
            uint32_t last_parity[C::STAGES];
            bool issued[C::STAGES];
            for (int s = 0; s < C::STAGES; ++s) issued[s] = false, last_parity[s] = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                SwapJob j;
                swap_job(args, t, nkb, j);
                const CUtensorMap* wmap = j.second ? &tmW2 : &tmW;
                for (int kb = j.kb0; kb < j.kb1; ++kb, ++kc) {
                    const int s = kc % C::STAGES;
                    const uint32_t ph = (kc / C::STAGES) & 1;
                    uint8_t* st = smem + s * C::STAGE_BYTES;
                    const bool x2 = args.k_wrap > 0 && kb * C::BK >= args.k_wrap;
                    const int kx = x2 ? kb * C::BK - args.k_wrap : kb * C::BK;
                    if (kc >= pre) {
                        if (!mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag, args.err, args.timeout_ns)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
                        tma_load_2d(st, wmap, &full[s], kx, j.wrow);
                        if (C::NA == 2) tma_load_2d(st + C::A_BYTES, wmap, &full[s], kx, j.wrow + args.up_offset);
                    }
                    tma_load_2d(st + C::NA * C::A_BYTES, x2 ? &tmX2 : &tmX, &full[s], kx, j.e.y);
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
            constexpr uint32_t idesc = umma_idesc_bf16(128, NT);
            uint32_t kc = 0;
            int it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++it) {
                const int buf = it & 1;
                const uint32_t use = (it >> 1) & 1;
                if (!mbar_wait_bounded(&tempty[buf], use ^ 1, abort_flag, args.err, args.timeout_ns)) break;
                tc_fence_after();
                const uint32_t d0 = tmem_base + buf * C::ACC_COLS;
                SwapJob j;
                swap_job(args, t, nkb, j);
                for (int kb = j.kb0; kb < j.kb1; ++kb, ++kc) {
                    const int s = kc % C::STAGES;
                    const uint32_t ph = (kc / C::STAGES) & 1;
                    if (!mbar_wait_bounded(&full[s], ph, abort_flag, args.err, args.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + s * C::STAGE_BYTES);
                    const uint64_t a0 = umma_desc_sw128(st);
                    const uint64_t a1 = umma_desc_sw128(st + C::A_BYTES);
                    const uint64_t bx = umma_desc_sw128(st + C::NA * C::A_BYTES);
#pragma unroll
                    for (int kk = 0; kk < C::BK / 16; ++kk) {
                        const uint32_t acc = (kb > j.kb0 || kk > 0) ? 1u : 0u;
                        umma_bf16(d0, a0 + 2 * kk, bx + 2 * kk, idesc, acc);
                        if (C::NA == 2) umma_bf16(d0 + NT, a1 + 2 * kk, bx + 2 * kk, idesc, acc);
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
            SwapJob j;
            swap_job(args, t, nkb, j);
            const int4 e = j.e;
            const int col = j.wt * 128 + quad * 32 + lane;
            const int buf = it & 1;
            const uint32_t use = (it >> 1) & 1;
            int ok = 1;
            if (lane == 0) ok = mbar_wait_bounded(&tfull[buf], use, abort_flag, args.err, args.timeout_ns) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + buf * C::ACC_COLS + (static_cast<uint32_t>(quad * 32) << 16);
            if (args.partial != nullptr) {
                // dense split-K projections: every token column's fp32 partial sum
                uint32_t g[NT];
                tmem_ld_cols<NT>(taddr, g);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[buf]);  // accumulator copied to registers: release it early
                if (col < args.part_rows) {
                    float4* dst = reinterpret_cast<float4*>(
                        args.partial + (static_cast<size_t>(j.split) * args.part_rows + col) * NT);
#pragma unroll
                    for (int i = 0; i < NT / 4; ++i)
                        dst[i] = make_float4(__uint_as_float(g[4 * i]), __uint_as_float(g[4 * i + 1]),
                                             __uint_as_float(g[4 * i + 2]), __uint_as_float(g[4 * i + 3]));
                }
            } else {
                // experts: only the expert's rows in this tile (e.z, the same for the whole warp), one at a time,
                // each row's accumulator column(s) read from tensor memory.  A small loop keeps the epilogue's
                // code small, so the TMA and MMA warps do not stall on instruction fetch.
                __nv_bfloat16* dst = args.out + static_cast<size_t>(e.y) * args.ld_out + col;
                for (int r = 0; r < e.z; ++r) {
                    uint32_t gv, uv = 0u;
                    tmem_ld_32x32b_x1(taddr + r, gv);
                    if (C::NA == 2) tmem_ld_32x32b_x1(taddr + NT + r, uv);
                    tmem_ld_wait();
                    float v = __uint_as_float(gv);
                    if (EPI == EPI_RELU2) v = act_relu2(v);
                    if (EPI == EPI_SWIGLU) v = act_silu_mul(v, __uint_as_float(uv));
                    if (col < args.n_out) dst[static_cast<size_t>(r) * args.ld_out] = __float2bfloat16_rn(v);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[buf]);  // this tile's accumulator is free for the MMA warp
            }
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

// Sum of the K splits in split order, then the epilogue, for the dense
// few-token projections.  One thread per (output column n, token t), n fastest.
//   n < n0:             out0[t][n] = bf16(act(sum) (+ resid[t][n] when resid is set)), partial row n
//   n0 <= n < n0 + n1:  out1[t][n - n0] = sum (fp32 router logits), partial row p1 + (n - n0)
// ACT: EPI_BF16 (none), EPI_RELU2, or EPI_SWIGLU (gate = partial row n, up =
// partial row up_row0 + n).  out0_lo (optional, ACT = EPI_BF16 without resid):
// out0_lo[t][n] = bf16(sum - bf16(sum)), the low part of the fp32 sum.
template <int NT, int ACT>
__global__ void __launch_bounds__(256) swap_reduce_kernel(const float* __restrict__ partial, int part_rows, int splits,
                                                          int T, int n0, int n1, int p1, int up_row0,
                                                          __nv_bfloat16* __restrict__ out0, int ld0,
                                                          float* __restrict__ out1, int ld1,
                                                          const __nv_bfloat16* __restrict__ resid, int ld_resid,
                                                          __nv_bfloat16* __restrict__ out0_lo) {
    pdl_begin();
    const long i = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int cols = n0 + n1;
    if (i >= static_cast<long>(cols) * T) return;
    const int n = static_cast<int>(i % cols), t = static_cast<int>(i / cols);
    const int prow = n < n0 ? n : p1 + (n - n0);
    // all split loads issue together; the sum is still taken in split order
    float pv[16];
#pragma unroll
    for (int s = 0; s < 16; ++s) pv[s] = s < splits ? partial[(static_cast<size_t>(s) * part_rows + prow) * NT + t] : 0.f;
    float v = 0.f;
#pragma unroll
    for (int s = 0; s < 16; ++s)
        if (s < splits) v += pv[s];
    if (ACT == EPI_RELU2 && n < n0) v = act_relu2(v);
    if (ACT == EPI_SWIGLU && n < n0) {
        float u = 0.f;
        for (int s = 0; s < splits; ++s) u += partial[(static_cast<size_t>(s) * part_rows + up_row0 + n) * NT + t];
        v = act_silu_mul(v, u);
    }
    if (n < n0) {
        if (resid != nullptr) v += __bfloat162float(resid[static_cast<size_t>(t) * ld_resid + n]);
        const __nv_bfloat16 hi = __float2bfloat16_rn(v);
        out0[static_cast<size_t>(t) * ld0 + n] = hi;
        if (out0_lo != nullptr) out0_lo[static_cast<size_t>(t) * ld0 + n] = __float2bfloat16_rn(v - __bfloat162float(hi));
    } else {
        out1[static_cast<size_t>(t) * ld1 + (n - n0)] = v;
    }
}

}  // namespace lmoe
