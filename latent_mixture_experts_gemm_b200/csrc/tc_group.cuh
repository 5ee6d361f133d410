// tc_group.cuh -- grouped expert GEMMs on CTA pairs, computed transposed.
//
// The expert GEMMs of a prefill batch are Y_e[rows_e x n] = X_e[rows_e x K] *
// W_e[n x K]^T for each expert e, with rows_e a few hundred and uneven.  A
// CTA-pair MMA (cta_group::2, M = 256) halves the operand bytes each SM loads
// per multiply-add against a single-CTA 128-row tile, but its 256 M rows must
// share one B operand.  Taking the expert's weight rows as the M operand makes
// that always true: every expert has n = m (or latent) weight rows, a multiple
// of 256.  The expert's token rows become the N operand, any multiple of 16 up
// to 256, so an expert with 352 rows is one N = 256 tile and one N = 96 tile,
// with no padding to 256 rows:
//
//   D^T[256 weight rows x N tokens] = W_e[256 x K] * X_e[N x K]^T
//
// Each CTA of the pair loads its own 128 weight rows and half of the N token
// rows (one box of 32, 64 or 128 rows), so an SM brings in 16 KB + N x 64 B
// per 64-deep K stage.  One thread of the first CTA issues the MMAs; each CTA's tensor
// memory receives its 128 weight rows x N tokens.  The epilogue thread is an
// output column (a weight row), its registers are tokens: eight warps per CTA,
// two per 32-lane quarter of tensor memory taking alternate 32-token blocks,
// apply the activation, transpose each 32 x 32 block through shared memory
// and write it with a TMA store; a block with fewer than 32 valid tokens (an
// expert's last) is stored row by row.  Each CTA's epilogue writes as many
// outputs per tile as a single-CTA 128 x 256 tile's, in half the main-loop
// time, hence the second set of epilogue warps.
//
// SwiGLU: each CTA's 128 weight rows are 16-row groups of gate rows and the
// matching up rows, alternating (one 5-D TMA box: K x 16 rows x {gate, up} x
// 4 groups x 1 expert), so lane l < 16 of a warp holds the gate of the
// feature whose up sits in lane l + 16: a shuffle pairs them, and the CTA
// writes 64 output features.
//
// Work list: entries {expert, first row, rows <= 256} (the counting sort's
// CTA-pair list).  Tile t = (entry t / n_mt, 256-row weight tile t % n_mt):
// consecutive tiles share their token rows.
//
// Synchronisation is that of the dense CTA-pair GEMM: full[s] on the first
// CTA collects both CTAs' bytes, empty[s] and tfull[b] are signalled to both
// CTAs by the MMA commit, tempty[b] on the first CTA counts the 16 epilogue
// warps of the pair.  Every wait is bounded.
#pragma once
#include "tc_gemm.cuh"

namespace lmoe {

struct GroupArgs {
    int K;                  // reduction length, multiple of 64
    int n_mt;               // 256-row weight tiles per expert (gated: 128 gate + 128 up rows per tile)
    const int4* list;       // {expert, first row, rows (1..256), 0}
    const int* count;       // entries of `list` (device)
    int w_rows_per_expert;  // weight rows per expert
    int up_offset;          // SwiGLU: row offset of the up rows inside an expert
    __nv_bfloat16* out;     // [rows, ld_out] bf16 outputs (the sorted row order of the inputs)
    int ld_out;
    int* err;
    unsigned long long timeout_ns;
};

struct GroupCfg {
    static constexpr int BK = 64;
    static constexpr int A_BYTES = 128 * BK * 2;  // this CTA's 128 weight rows
    static constexpr int B_BYTES = 128 * BK * 2;  // room for this CTA's half of up to 256 token rows
    static constexpr int STAGES = 6;
    static constexpr int TMEM_COLS = 512;         // two accumulators of up to 256 token columns
    static constexpr int EPI_WARPS = 8;
    static constexpr int THREADS = 64 + 32 * EPI_WARPS;
    static constexpr int OUT_BYTES = EPI_WARPS * 2 * 2048; // per epilogue warp: two 32 x 32 bf16 staging blocks
    static constexpr int SMEM_BYTES = STAGES * (A_BYTES + B_BYTES) + OUT_BYTES + 1024 + 256;
    static_assert(SMEM_BYTES <= 232448, "shared memory");
};

struct GroupJob {
    int expert, row0, rows;  // the entry's expert and token rows
    int n;                   // MMA N: rows rounded up to 16
    int mt;                  // 256-row weight tile of the expert
};

__device__ __forceinline__ void group_job(const GroupArgs& a, int t, GroupJob& j) {
    const int4 e = a.list[t / a.n_mt];
    j.mt = t % a.n_mt;
    j.expert = e.x;
    j.row0 = e.y;
    j.rows = e.z;
    j.n = max(16, (e.z + 15) & ~15);
}

// Instruction descriptor of a bf16 pair MMA with a run-time N (fp32 accumulate, both K-major).
__device__ __forceinline__ uint32_t idesc_bf16_m256(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (16u << 24);
}

template <int EPI>
__global__ void __launch_bounds__(GroupCfg::THREADS, 1)
    tc_group_pair_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX32,
                         const __grid_constant__ CUtensorMap tmX64, const __grid_constant__ CUtensorMap tmX128,
                         const __grid_constant__ CUtensorMap tmOut, const GroupArgs args) {
    pdl_begin();
    using C = GroupCfg;
    constexpr bool GATED = EPI == EPI_SWIGLU;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + C::STAGES * C::A_BYTES;
    uint8_t* sOut = sB + C::STAGES * C::B_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(sOut + C::OUT_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* tfull = empty + C::STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int pid = static_cast<int>(blockIdx.x >> 1), npid = static_cast<int>(gridDim.x >> 1);
    const int ntiles = (*args.count) * args.n_mt;
    if (pid >= ntiles) return;  // both CTAs of the pair leave together, before any pair set-up

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 2 * C::EPI_WARPS);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmX32);
        tma_prefetch_desc(&tmX64);
        tma_prefetch_desc(&tmX128);
        tma_prefetch_desc(&tmOut);
    }
    if (warp == 1) tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // both CTAs' barriers initialised before any copy or arrive reaches them
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int nkb = args.K / C::BK;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer (both CTAs)
            uint32_t kc = 0;
            uint32_t last_parity[C::STAGES];
            bool issued[C::STAGES];
            for (int s = 0; s < C::STAGES; ++s) issued[s] = false, last_parity[s] = 0;
            bool ok = true;
            for (int t = pid; t < ntiles && ok; t += npid) {
                GroupJob j;
                group_job(args, t, j);
                const int wbase = j.expert * args.w_rows_per_expert;
                const int half = j.n >> 1;  // token rows of this CTA, loaded as one box of 32, 64 or 128 rows
                const int box = half <= 32 ? 32 : (half <= 64 ? 64 : 128);
                const CUtensorMap* xmap = half <= 32 ? &tmX32 : (half <= 64 ? &tmX64 : &tmX128);
                const int xrow = j.row0 + static_cast<int>(rank) * half;
                const uint32_t bytes = 2u * (C::A_BYTES + box * C::BK * 2);  // both CTAs
                for (int kb = 0; kb < nkb; ++kb, ++kc) {
                    const int s = kc % C::STAGES;
                    const uint32_t ph = (kc / C::STAGES) & 1;
                    if (!mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag, args.err, args.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], bytes);
                    const uint32_t fb = mapa_shared(&full[s], 0);
                    uint8_t* a = sA + s * C::A_BYTES;
                    if (GATED) {
                        // 4 groups of 16 features: gate rows of features f .. f+15, then their up rows
                        const int g0 = (j.mt * 128 + 64 * static_cast<int>(rank)) / 16;
                        tma_load_5d_pair(a, &tmW, fb, kb * C::BK, 0, 0, g0, j.expert);
                    } else {
                        tma_load_2d_pair(a, &tmW, fb, kb * C::BK, wbase + j.mt * 256 + 128 * static_cast<int>(rank));
                    }
                    tma_load_2d_pair(sB + s * C::B_BYTES, xmap, fb, kb * C::BK, xrow);
                    issued[s] = true;
                    last_parity[s] = ph;
                }
            }
            if (rank == 0)
                for (int s = 0; s < C::STAGES; ++s)
                    if (issued[s]) {
                        int no_abort = 0;
                        const uint64_t drain = args.timeout_ns > 200000000ull ? args.timeout_ns : 200000000ull;
                        mbar_wait_bounded(&full[s], last_parity[s], &no_abort, args.err, drain);
                    }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ------------------------------------------------ MMA issuer (first CTA)
            uint32_t kc = 0;
            int it = 0;
            bool ok = true;
            for (int t = pid; t < ntiles && ok; t += npid, ++it) {
                GroupJob j;
                group_job(args, t, j);
                const uint32_t idesc = idesc_bf16_m256(j.n);
                const int buf = it & 1;
                const uint32_t use = (it >> 1) & 1;
                if (!mbar_wait_bounded(&tempty[buf], use ^ 1, abort_flag, args.err, args.timeout_ns)) break;
                tc_fence_after();
                const uint32_t dtmem = tmem_base + buf * 256;
                for (int kb = 0; kb < nkb; ++kb, ++kc) {
                    const int s = kc % C::STAGES;
                    const uint32_t ph = (kc / C::STAGES) & 1;
                    if (!mbar_wait_bounded(&full[s], ph, abort_flag, args.err, args.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = umma_desc_sw128(smem_u32(sA + s * C::A_BYTES));
                    const uint64_t bd = umma_desc_sw128(smem_u32(sB + s * C::B_BYTES));
#pragma unroll
                    for (int kk = 0; kk < C::BK / 16; ++kk)
                        umma_bf16_pair(dtmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    umma_commit_pair_mc(&empty[s], 0x3);
                }
                if (ok) umma_commit_pair_mc(&tfull[buf], 0x3);
            }
            umma_commit_pair(mma_done);
            int no_abort = 0;
            const uint64_t drain = args.timeout_ns > 200000000ull ? args.timeout_ns : 200000000ull;
            mbar_wait_bounded(mma_done, 0, &no_abort, args.err, drain);
        }
    } else {
        // ---------------------------------------------------- epilogue (both CTAs): thread = weight row
        const int quad = warp & 3;                  // the 32-lane quarter of tensor memory this warp may read
        const int sub = (warp - 2) >> 2;            // which of the quarter's two warps: alternate 32-token blocks
        uint8_t* stage = sOut + (warp - 2) * 4096;  // this warp's two 2 KB staging blocks
        uint32_t sbuf = 0;
        int it = 0;
        for (int t = pid; t < ntiles; t += npid, ++it) {
            GroupJob j;
            group_job(args, t, j);
            const int buf = it & 1;
            const uint32_t use = (it >> 1) & 1;
            int ok = 1;
            if (lane == 0) ok = mbar_wait_bounded(&tfull[buf], use, abort_flag, args.err, args.timeout_ns) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + buf * 256 + (static_cast<uint32_t>(quad * 32) << 16);
            // output features of this warp: 32 (16 gated) consecutive columns starting at fw
            const int fw = GATED ? j.mt * 128 + 64 * static_cast<int>(rank) + 16 * quad
                                 : j.mt * 256 + 128 * static_cast<int>(rank) + 32 * quad;
            // 32-token blocks c0 = 32 sub, 32 sub + 64, ...: the next block's tensor-memory load is issued
            // before this block is staged and stored, so it overlaps them
            int c0 = 32 * sub;
            uint32_t v[32];
            if (c0 < j.rows) {
                tmem_ld_32x32b_x32(tbase + c0, v);
                tmem_ld_wait();
            }
#pragma unroll 1
            for (; c0 < j.rows; c0 += 64) {
                const int valid = min(32, j.rows - c0);
                const size_t orow = static_cast<size_t>(j.row0) + c0;
                const bool more = c0 + 64 < j.rows;
                if (!GATED) {
                    __nv_bfloat16 h[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        float x = __uint_as_float(v[i]);
                        if (EPI == EPI_RELU2) x = act_relu2(x);
                        h[i] = __float2bfloat16_rn(x);
                    }
                    if (more) tmem_ld_32x32b_x32(tbase + c0 + 64, v);
                    if (valid == 32) {
                        staging_acquire(lane);
                        __nv_bfloat16* sb = reinterpret_cast<__nv_bfloat16*>(stage + sbuf * 2048);
#pragma unroll
                        for (int i = 0; i < 32; ++i) sb[i * 32 + lane] = h[i];  // [token][feature]
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tmOut, sb, fw, static_cast<int>(orow));
                            bulk_commit_group();
                        }
                        sbuf ^= 1u;
                    } else {
                        __nv_bfloat16* dst = args.out + orow * args.ld_out + fw + lane;
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (i < valid) dst[static_cast<size_t>(i) * args.ld_out] = h[i];
                    }
                } else {
                    // lane l < 16: gate of feature fw + l for tokens c0 .. c0+31; lane l + 16: its up.
                    // Each lane keeps 16 tokens: lane l the first 16, lane l + 16 the last 16.
                    const bool lo = lane < 16;
                    __nv_bfloat16 h[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const uint32_t send = lo ? v[16 + i] : v[i];
                        const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, 16);
                        const float g = __uint_as_float(lo ? v[i] : recv);
                        const float u = __uint_as_float(lo ? recv : v[16 + i]);
                        h[i] = __float2bfloat16_rn(act_silu_mul(g, u));
                    }
                    if (more) tmem_ld_32x32b_x32(tbase + c0 + 64, v);
                    const int tok0 = lo ? 0 : 16;
                    const int f = lane & 15;
                    if (valid == 32) {
                        staging_acquire(lane);
                        __nv_bfloat16* sb = reinterpret_cast<__nv_bfloat16*>(stage + sbuf * 2048);
#pragma unroll
                        for (int i = 0; i < 16; ++i) sb[(tok0 + i) * 16 + f] = h[i];  // [token][16 features]
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tmOut, sb, fw, static_cast<int>(orow));
                            bulk_commit_group();
                        }
                        sbuf ^= 1u;
                    } else {
                        __nv_bfloat16* dst = args.out + orow * args.ld_out + fw + f;
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (tok0 + i < valid) dst[static_cast<size_t>(tok0 + i) * args.ld_out] = h[i];
                    }
                }
                if (more) tmem_ld_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(&tempty[buf], 0));
        }
        if (lane == 0) bulk_wait_group_all();
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace lmoe
