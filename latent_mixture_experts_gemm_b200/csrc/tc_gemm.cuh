// tc_gemm.cuh -- persistent tcgen05 GEMM for sm_100a: D[128 x BN] tiles of A[M,K] * B[N,K]^T.
//
// Both operands are bf16 and K-major (rows contiguous along K); TMA brings
// 128 x 64 A tiles and BN x 64 B tiles into shared memory with the 128-byte
// swizzle; one thread issues tcgen05.mma (M=128, N=BN, K=16) into a tensor
// memory accumulator; four epilogue warps read the accumulator back with
// tcgen05.ld and apply the fused epilogue.  Two accumulators (2 x BN TMEM
// columns) let the epilogue of tile i overlap the main loop of tile i+1.
//
// Warp roles (192 threads): warp 0 = TMA producer, warp 1 = TMEM owner and MMA
// issuer, warps 2..5 = epilogue (warp w reads TMEM lanes 32*(w%4) .. +31).
//
// Tile maps:
//   dense   -- tiles over ceil(M/128) x n_tiles, n fastest (CTAs working at
//              the same time share the A rows through L2);
//   grouped -- an M-tile list built on the device (expert, first row, rows);
//              tile t -> list entry t / n_tiles, column tile t % n_tiles; the
//              B rows are those of the entry's expert.
#pragma once
#include "ptx.cuh"

namespace lmoe {

enum Epi : int {
    EPI_BF16 = 0,         // out0 = bf16(acc)
    EPI_RELU2 = 1,        // out0 = bf16(relu(acc)^2)
    EPI_SWIGLU = 2,       // accumulator columns [0,BN/2) gate, [BN/2,BN) up: out0 = bf16(silu(g) * u)
    EPI_RESID = 3,        // out0 = bf16(acc + resid)
    EPI_PROJ_ROUTER = 4,  // column tiles < n_tiles0: bf16 -> out0; the rest: fp32 -> out1 (masked to N1)
};

struct GemmArgs {
    int M;                 // dense: rows of A
    int K;                 // reduction length, multiple of 64
    int n_tiles;           // column tiles per M-tile
    int n_tiles0;          // EPI_PROJ_ROUTER: column tiles of segment 0
    int N0;                // valid output columns of out0 (segment 0)
    int N1;                // EPI_PROJ_ROUTER: valid columns of out1
    const int4* mt_list;   // grouped: {expert, first row, rows, 0}; nullptr => dense
    const int* mt_count;   // grouped: number of list entries (device)
    int b_rows_per_expert; // grouped: rows of B per expert
    int up_offset;         // EPI_SWIGLU: row offset of the up half inside an expert
    __nv_bfloat16* out0;
    int ld0;
    float* out1;
    int ld1;
    const __nv_bfloat16* resid;
    int ld_resid;
    int tma_store;         // 1: bf16 out0 rows leave through shared-memory staging and TMA stores (BN = 256)
    // Two-part A: with k_wrap > 0 the reduction runs over K = 2 * k_wrap; k-blocks at or past k_wrap take
    // their A tile from tmA2 and their B tile from k - k_wrap, so the product is (A + A2) * B^T with B read
    // twice.  A bf16 split A = hi + lo of an fp32 operand then multiplies at ~16 significant bits.
    int k_wrap;
    // EPI_BF16 without TMA stores: also write out_lo = bf16(acc - bf16(acc)), the low part of the fp32
    // accumulator (ld0 is its row pitch too)
    __nv_bfloat16* out_lo;
    int* err;
    unsigned long long timeout_ns;
};

// Output staging for TMA stores: each epilogue warp owns two 4 KB buffers of 32 rows x 64 bf16
// columns.  Row r sits at r * 128 bytes with its 16-byte chunk c at position c ^ (r % 8): the
// 128-byte swizzle of the output map (buffers are 1024-byte aligned).
constexpr int OUT_STAGE_BYTES = 4 * 2 * 32 * 128;

template <int BN>
struct GemmCfg {
    static constexpr int BM = 128;
    static constexpr int BK = 64;
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGES = (BN >= 256) ? 4 : (BN >= 128 ? 6 : 8);
    static constexpr int TMEM_COLS = 2 * BN;  // power of two for BN in {64,128,256}
    static constexpr int SMEM_BYTES =
        STAGES * (A_BYTES + B_BYTES) + OUT_STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
};

struct TileJob {
    int a_row0, rows;   // A rows (and output rows) of this tile
    int b_row0, b_row1; // B rows of the (first, second) half
    int col0;           // first output column
    int seg;            // EPI_PROJ_ROUTER: 0 latent columns, 1 router columns
};

template <int BN, int EPI>
__device__ __forceinline__ void tile_job(const GemmArgs& a, int t, TileJob& j) {
    const int mt = t / a.n_tiles, nt = t % a.n_tiles;
    j.seg = 0;
    if (a.mt_list != nullptr) {
        const int4 e = a.mt_list[mt];
        j.a_row0 = e.y;
        j.rows = e.z;
        if (EPI == EPI_SWIGLU) {
            j.col0 = nt * (BN / 2);
            j.b_row0 = e.x * a.b_rows_per_expert + j.col0;
            j.b_row1 = j.b_row0 + a.up_offset;
        } else {
            j.col0 = nt * BN;
            j.b_row0 = e.x * a.b_rows_per_expert + j.col0;
            j.b_row1 = 0;
        }
    } else {
        j.a_row0 = mt * 128;
        j.rows = min(128, a.M - j.a_row0);
        if (EPI == EPI_PROJ_ROUTER && nt >= a.n_tiles0) {
            j.seg = 1;
            j.col0 = (nt - a.n_tiles0) * BN;
        } else {
            j.col0 = (EPI == EPI_SWIGLU) ? nt * (BN / 2) : nt * BN;
        }
        j.b_row0 = j.col0;
        j.b_row1 = j.col0 + a.up_offset;
    }
}

template <int BN>
__device__ __forceinline__ int total_tiles(const GemmArgs& a) {
    if (a.mt_list != nullptr) return (*a.mt_count) * a.n_tiles;
    return ((a.M + 127) / 128) * a.n_tiles;
}

// Bound of the waits that drain in-flight copies and MMAs before the CTA
// exits: never shorter than 200 ms, whatever the configured wait bound.
__device__ __forceinline__ uint64_t drain_ns(const GemmArgs& a) {
    return a.timeout_ns > 200000000ull ? a.timeout_ns : 200000000ull;
}

__device__ __forceinline__ float act_relu2(float v) {
    const float r = fmaxf(v, 0.0f);
    return r * r;
}
__device__ __forceinline__ float act_silu_mul(float g, float u) { return g / (1.0f + expf(-g)) * u; }

// Residual of 64 output columns starting at pair column `pc` of the tile (zeros where not needed).
template <int BN>
__device__ __forceinline__ void epi_load_resid(const GemmArgs& a, const TileJob& j, int pc, bool row_ok, size_t row,
                                               uint4 (&rs)[8]) {
    const int col = j.col0 + pc;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const bool ok = row_ok && col + 32 * h < a.N0;
        const uint4* src = reinterpret_cast<const uint4*>(a.resid + row * a.ld_resid + col + 32 * h);
#pragma unroll
        for (int i = 0; i < 4; ++i) rs[4 * h + i] = ok ? src[i] : make_uint4(0, 0, 0, 0);
    }
}

__device__ __forceinline__ void stage_row64(uint8_t* buf, int lane, const uint4 (&q)[8]) {
    uint8_t* rowp = buf + lane * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(rowp + ((c ^ (lane & 7)) << 4)) = q[c];
}

// Hand this warp's staged 32 x 64 block to the TMA unit once every lane has written it.
__device__ __forceinline__ void store_block64(const CUtensorMap* map, const uint8_t* buf, int lane, int col, int row0) {
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(map, buf, col, row0);
        bulk_commit_group();
    }
}

// Before rewriting a staging buffer: the store issued from it one block earlier has read it.
__device__ __forceinline__ void staging_acquire(int lane) {
    if (lane == 0) bulk_wait_group_read<1>();
    __syncwarp();
}

__device__ __forceinline__ uint4 pack8(const float* f) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
}

// Epilogue of one tile for the 128 accumulator rows of this CTA: warp w (w % 4 = quad) reads TMEM
// lanes 32*quad .. +31 at `tbase`, applies the fused epilogue and stores row `row` (when row_ok).
// For EPI_RESID, `rs` holds the residual of the first 64 columns on entry.  With `tma_rows` (all
// 32 rows of this warp valid, and a bf16 output map), the bf16 outputs go out in 64-column blocks
// through this warp's staging buffers `sout` and TMA stores to `tmOut` at rows warp_row0 ..;
// otherwise every thread stores its own row.
template <int BN, int EPI>
__device__ __forceinline__ void gemm_epilogue_store(const GemmArgs& args, const TileJob& j, bool row_ok, size_t row,
                                                    uint32_t tbase, uint4 (&rs)[8], const CUtensorMap* tmOut,
                                                    uint8_t* sout, uint32_t& sbuf, bool tma_rows, int warp_row0,
                                                    int lane) {
    if (EPI == EPI_SWIGLU) {
        uint32_t pk_prev[16];
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
            uint32_t g[32], u[32];
            tmem_ld_32x32b_x32(tbase + c, g);
            tmem_ld_32x32b_x32(tbase + BN / 2 + c, u);
            tmem_ld_wait();
            const int col = j.col0 + c;
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                pk[i] = pack_bf16x2(act_silu_mul(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                                    act_silu_mul(__uint_as_float(g[2 * i + 1]), __uint_as_float(u[2 * i + 1])));
            if (tma_rows) {
                if ((c & 32) == 0) {  // first half of a 64-column block
#pragma unroll
                    for (int i = 0; i < 16; ++i) pk_prev[i] = pk[i];
                } else if (col - 32 < args.N0) {
                    uint4 q[8];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        q[i] = make_uint4(pk_prev[4 * i], pk_prev[4 * i + 1], pk_prev[4 * i + 2], pk_prev[4 * i + 3]);
                        q[4 + i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                    }
                    staging_acquire(lane);
                    uint8_t* buf = sout + sbuf * 4096;
                    stage_row64(buf, lane, q);
                    store_block64(tmOut, buf, lane, col - 32, warp_row0);
                    sbuf ^= 1u;
                }
            } else if (row_ok && col < args.N0) {
                uint4* dst = reinterpret_cast<uint4*>(args.out0 + row * args.ld0 + col);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
        }
    } else {
        // 64 accumulator columns per tcgen05 wait
#pragma unroll 1
        for (int pc = 0; pc < BN; pc += 64) {
            uint32_t v2[2][32];
            tmem_ld_32x32b_x32(tbase + pc, v2[0]);
            tmem_ld_32x32b_x32(tbase + pc + 32, v2[1]);
            uint4 rs_now[8];
            if (EPI == EPI_RESID) {
#pragma unroll
                for (int i = 0; i < 8; ++i) rs_now[i] = rs[i];
                if (pc + 64 < BN) epi_load_resid<BN>(args, j, pc + 64, row_ok, row, rs);
            }
            tmem_ld_wait();
            if (!row_ok) continue;  // (with tma_rows every lane's row is valid: no divergence)
            const int col = j.col0 + pc;
            if (EPI == EPI_PROJ_ROUTER && j.seg == 1) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t(&v)[32] = v2[h];
                    const int ch = col + 32 * h;
                    float* dst = args.out1 + row * args.ld1 + ch;
                    if (ch + 32 <= args.N1) {
                        float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            d4[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                                __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (ch + i < args.N1) dst[i] = __uint_as_float(v[i]);
                    }
                }
                continue;
            }
            if (col >= args.N0) continue;
            uint4 q[8];
            const bool lo_out = EPI == EPI_BF16 && args.out_lo != nullptr && !tma_rows;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float f[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v2[h][i]);
                if (lo_out) {
                    // the rounding error of each bf16 output, exact in fp32, itself stored in bf16
                    float r[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = f[i] - __bfloat162float(__float2bfloat16_rn(f[i]));
                    uint4* dlo = reinterpret_cast<uint4*>(args.out_lo + row * args.ld0 + col + 32 * h);
#pragma unroll
                    for (int i = 0; i < 4; ++i) dlo[i] = pack8(r + 8 * i);
                }
                if (EPI == EPI_RELU2) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) f[i] = act_relu2(f[i]);
                }
                if (EPI == EPI_RESID) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint4 r4 = rs_now[4 * h + i];
                        f[8 * i + 0] += bf16lo(r4.x);
                        f[8 * i + 1] += bf16hi(r4.x);
                        f[8 * i + 2] += bf16lo(r4.y);
                        f[8 * i + 3] += bf16hi(r4.y);
                        f[8 * i + 4] += bf16lo(r4.z);
                        f[8 * i + 5] += bf16hi(r4.z);
                        f[8 * i + 6] += bf16lo(r4.w);
                        f[8 * i + 7] += bf16hi(r4.w);
                    }
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) q[4 * h + i] = pack8(f + 8 * i);
            }
            if (tma_rows) {
                staging_acquire(lane);
                uint8_t* buf = sout + sbuf * 4096;
                stage_row64(buf, lane, q);
                store_block64(tmOut, buf, lane, col, warp_row0);
                sbuf ^= 1u;
            } else {
                uint4* dst = reinterpret_cast<uint4*>(args.out0 + row * args.ld0 + col);
#pragma unroll
                for (int i = 0; i < 8; ++i) dst[i] = q[i];
            }
        }
    }
}

template <int BN, int EPI>
__global__ void __launch_bounds__(192, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmOut,
                   const __grid_constant__ CUtensorMap tmA2, const GemmArgs args) {
    pdl_begin();
    using C = GemmCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + C::STAGES * C::A_BYTES;
    uint8_t* sOut = sB + C::STAGES * C::B_BYTES;  // epilogue staging (1024-aligned)
    uint64_t* full = reinterpret_cast<uint64_t*>(sOut + OUT_STAGE_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* tfull = empty + C::STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = total_tiles<BN>(args);
    if (static_cast<int>(blockIdx.x) >= ntiles) return;  // no tile for this CTA: skip TMEM and barrier set-up

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
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (EPI == EPI_PROJ_ROUTER) tma_prefetch_desc(&tmB2);
        if (args.k_wrap > 0) tma_prefetch_desc(&tmA2);
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int nkb = args.K / C::BK;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            uint32_t kc = 0;
            uint32_t last_parity[C::STAGES];
            bool issued[C::STAGES];
            for (int s = 0; s < C::STAGES; ++s) issued[s] = false, last_parity[s] = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                TileJob j;
                tile_job<BN, EPI>(args, t, j);
                const CUtensorMap* bmap = (EPI == EPI_PROJ_ROUTER && j.seg == 1) ? &tmB2 : &tmB;
                for (int kb = 0; kb < nkb; ++kb, ++kc) {
                    const int s = kc % C::STAGES;
                    const uint32_t ph = (kc / C::STAGES) & 1;
                    if (!mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag, args.err, args.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    const bool a2 = args.k_wrap > 0 && kb * C::BK >= args.k_wrap;
                    const int kx = a2 ? kb * C::BK - args.k_wrap : kb * C::BK;
                    mbar_arrive_expect_tx(&full[s], C::A_BYTES + C::B_BYTES);
                    tma_load_2d(sA + s * C::A_BYTES, a2 ? &tmA2 : &tmA, &full[s], kx, j.a_row0);
                    if (EPI == EPI_SWIGLU) {
                        tma_load_2d(sB + s * C::B_BYTES, bmap, &full[s], kx, j.b_row0);
                        tma_load_2d(sB + s * C::B_BYTES + C::B_BYTES / 2, bmap, &full[s], kx, j.b_row1);
                    } else {
                        tma_load_2d(sB + s * C::B_BYTES, bmap, &full[s], kx, j.b_row0);
                    }
                    issued[s] = true;
                    last_parity[s] = ph;
                }
            }
            // Never leave a copy in flight into shared memory: wait for the last
            // load issued on each stage (immediate when it was consumed).
            for (int s = 0; s < C::STAGES; ++s)
                if (issued[s]) {
                    int no_abort = 0;
                    mbar_wait_bounded(&full[s], last_parity[s], &no_abort, args.err, drain_ns(args));
                }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            constexpr uint32_t idesc = umma_idesc_bf16(128, BN);
            uint32_t kc = 0;
            int it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++it) {
                const int buf = it & 1;
                const uint32_t use = (it >> 1) & 1;
                if (!mbar_wait_bounded(&tempty[buf], use ^ 1, abort_flag, args.err, args.timeout_ns)) break;
                tc_fence_after();
                const uint32_t dtmem = tmem_base + buf * BN;
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
                        umma_bf16(dtmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&empty[s]);
                }
                if (ok) umma_commit(&tfull[buf]);
            }
            // Wait for every MMA this thread issued before TMEM can be released.
            umma_commit(mma_done);
            int no_abort = 0;
            mbar_wait_bounded(mma_done, 0, &no_abort, args.err, drain_ns(args));
        }
    } else {
        // ---------------------------------------------------- epilogue
        const int quad = warp & 3;
        const int row_in_tile = quad * 32 + lane;
        uint32_t sbuf = 0;
        int it = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
            TileJob j;
            tile_job<BN, EPI>(args, t, j);
            const int buf = it & 1;
            const uint32_t use = (it >> 1) & 1;
            const bool row_ok = row_in_tile < j.rows;
            const size_t row = static_cast<size_t>(j.a_row0) + row_in_tile;
            // The residual of the first 64 columns is requested before the accumulator
            // is ready; each later 64-column pair is requested one pair ahead.
            uint4 rs[8];
            if (EPI == EPI_RESID) epi_load_resid<BN>(args, j, 0, row_ok, row, rs);
            // One lane waits and the verdict is broadcast, so the whole warp
            // either reads the accumulator (tcgen05.ld is warp-collective) or leaves.
            int ok = 1;
            if (lane == 0) ok = mbar_wait_bounded(&tfull[buf], use, abort_flag, args.err, args.timeout_ns) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + buf * BN + (static_cast<uint32_t>(quad * 32) << 16);
            const bool tma_rows = BN == 256 && args.tma_store != 0 && j.rows >= quad * 32 + 32 &&
                                  !(EPI == EPI_PROJ_ROUTER && j.seg == 1);
            gemm_epilogue_store<BN, EPI>(args, j, row_ok, row, tbase, rs, &tmOut, sOut + quad * 8192, sbuf, tma_rows,
                                         j.a_row0 + quad * 32, lane);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[buf]);
        }
        if (lane == 0) bulk_wait_group_all();  // the tile stores are complete before the CTA can exit
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ============================================================================ CTA-pair GEMM
// The same GEMM on pairs of CTAs (a cluster of 2) issuing cta_group::2 MMAs:
// a pair tile is 256 rows x 256 columns.  Each CTA loads its own 128 A rows
// and half of the tile's B rows (128), so an SM brings in 32 KB per 64-deep K
// stage instead of 48 KB for the same multiply-adds: the operand bytes per MAC
// fall by a third, which is what bounds the single-CTA kernel (its operand
// loads are latency-bound).  One thread of the first CTA issues the MMAs; each
// CTA's tensor memory receives its own 128 rows of the 256 x 256 accumulator
// and its own epilogue stores them.
//
// Synchronisation of the pair:
//   full[s]   first CTA only: its producer posts the stage's bytes of both
//             CTAs; both CTAs' copies complete on it (its cluster address);
//   empty[s]  both CTAs: the MMA thread's commit arrives on both (multicast);
//   tfull[b]  both CTAs: the commit after a tile's last stage (multicast);
//   tempty[b] first CTA only: the 8 epilogue warps of both CTAs arrive on it.
// Every wait is bounded, so each thread reaches the cluster barrier before the
// CTAs free their tensor memory, even after a timeout.
//
// Tile maps: dense -- ceil(M/256) x n_tiles; grouped -- the pair list
// (expert, first row, rows <= 256).  For EPI_SWIGLU the first CTA loads the
// gate rows and the second the matching up rows, so accumulator columns
// [0,128) are gate and [128,256) up, as in the single-CTA kernel's layout.
struct GemmPairCfg {
    static constexpr int BN = 256;
    static constexpr int BK = 64;
    static constexpr int A_BYTES = 128 * BK * 2;       // this CTA's 128 A rows
    static constexpr int B_BYTES = (BN / 2) * BK * 2;  // this CTA's half of the B rows
    static constexpr int STAGES = 6;
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr int SMEM_BYTES = STAGES * (A_BYTES + B_BYTES) + OUT_STAGE_BYTES + 1024 + 256;
    static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <int EPI>
__device__ __forceinline__ void tile_job_pair(const GemmArgs& a, int t, int rank, TileJob& j) {
    const int mt = t / a.n_tiles, nt = t % a.n_tiles;
    int row0, rows;
    j.seg = 0;
    j.b_row1 = 0;
    if (a.mt_list != nullptr) {
        const int4 e = a.mt_list[mt];
        row0 = e.y;
        rows = e.z;
        const int base = e.x * a.b_rows_per_expert;
        if (EPI == EPI_SWIGLU) {
            j.col0 = nt * 128;
            j.b_row0 = base + j.col0 + (rank ? a.up_offset : 0);
        } else {
            j.col0 = nt * 256;
            j.b_row0 = base + j.col0 + 128 * rank;
        }
    } else {
        row0 = mt * 256;
        rows = min(256, a.M - row0);
        if (EPI == EPI_PROJ_ROUTER && nt >= a.n_tiles0) {
            j.seg = 1;
            j.col0 = (nt - a.n_tiles0) * 256;
        } else {
            j.col0 = (EPI == EPI_SWIGLU) ? nt * 128 : nt * 256;
        }
        j.b_row0 = (EPI == EPI_SWIGLU) ? j.col0 + (rank ? a.up_offset : 0) : j.col0 + 128 * rank;
    }
    j.a_row0 = row0 + 128 * rank;
    j.rows = max(0, min(128, rows - 128 * rank));
}

__device__ __forceinline__ int total_tiles_pair(const GemmArgs& a) {
    if (a.mt_list != nullptr) return (*a.mt_count) * a.n_tiles;
    return ((a.M + 255) / 256) * a.n_tiles;
}

template <int EPI>
__global__ void __launch_bounds__(192, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmOut,
                        const __grid_constant__ CUtensorMap tmA2, const GemmArgs args) {
    pdl_begin();
    using C = GemmPairCfg;
    constexpr int BN = C::BN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + C::STAGES * C::A_BYTES;
    uint8_t* sOut = sB + C::STAGES * C::B_BYTES;  // epilogue staging (1024-aligned)
    uint64_t* full = reinterpret_cast<uint64_t*>(sOut + OUT_STAGE_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* tfull = empty + C::STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int pid = static_cast<int>(blockIdx.x >> 1), npid = static_cast<int>(gridDim.x >> 1);
    const int ntiles = total_tiles_pair(args);
    if (pid >= ntiles) return;  // both CTAs of the pair leave together, before any pair set-up

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 8);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (EPI == EPI_PROJ_ROUTER) tma_prefetch_desc(&tmB2);
        if (args.k_wrap > 0) tma_prefetch_desc(&tmA2);
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
                TileJob j;
                tile_job_pair<EPI>(args, t, static_cast<int>(rank), j);
                const CUtensorMap* bmap = (EPI == EPI_PROJ_ROUTER && j.seg == 1) ? &tmB2 : &tmB;
                for (int kb = 0; kb < nkb; ++kb, ++kc) {
                    const int s = kc % C::STAGES;
                    const uint32_t ph = (kc / C::STAGES) & 1;
                    if (!mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag, args.err, args.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * (C::A_BYTES + C::B_BYTES));
                    const uint32_t fb = mapa_shared(&full[s], 0);
                    const bool a2 = args.k_wrap > 0 && kb * C::BK >= args.k_wrap;
                    const int kx = a2 ? kb * C::BK - args.k_wrap : kb * C::BK;
                    tma_load_2d_pair(sA + s * C::A_BYTES, a2 ? &tmA2 : &tmA, fb, kx, j.a_row0);
                    tma_load_2d_pair(sB + s * C::B_BYTES, bmap, fb, kx, j.b_row0);
                    issued[s] = true;
                    last_parity[s] = ph;
                }
            }
            // The first CTA's full barriers count both CTAs' bytes: waiting for the last phase of each
            // stage there means no copy of either CTA is still in flight.  The second CTA leaves only
            // after the final cluster barrier, which the first passes after this drain.
            if (rank == 0)
                for (int s = 0; s < C::STAGES; ++s)
                    if (issued[s]) {
                        int no_abort = 0;
                        mbar_wait_bounded(&full[s], last_parity[s], &no_abort, args.err, drain_ns(args));
                    }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ------------------------------------------------ MMA issuer (first CTA)
            constexpr uint32_t idesc = umma_idesc_bf16(256, BN);
            uint32_t kc = 0;
            int it = 0;
            bool ok = true;
            for (int t = pid; t < ntiles && ok; t += npid, ++it) {
                const int buf = it & 1;
                const uint32_t use = (it >> 1) & 1;
                if (!mbar_wait_bounded(&tempty[buf], use ^ 1, abort_flag, args.err, args.timeout_ns)) break;
                tc_fence_after();
                const uint32_t dtmem = tmem_base + buf * BN;
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
            // every MMA of the pair done before the tensor memory of either CTA is freed
            umma_commit_pair(mma_done);
            int no_abort = 0;
            mbar_wait_bounded(mma_done, 0, &no_abort, args.err, drain_ns(args));
        }
    } else {
        // ---------------------------------------------------- epilogue (both CTAs, own 128 rows)
        const int quad = warp & 3;
        const int row_in_tile = quad * 32 + lane;
        uint32_t sbuf = 0;
        int it = 0;
        for (int t = pid; t < ntiles; t += npid, ++it) {
            TileJob j;
            tile_job_pair<EPI>(args, t, static_cast<int>(rank), j);
            const int buf = it & 1;
            const uint32_t use = (it >> 1) & 1;
            const bool row_ok = row_in_tile < j.rows;
            const size_t row = static_cast<size_t>(j.a_row0) + row_in_tile;
            uint4 rs[8];
            if (EPI == EPI_RESID) epi_load_resid<BN>(args, j, 0, row_ok, row, rs);
            int ok = 1;
            if (lane == 0) ok = mbar_wait_bounded(&tfull[buf], use, abort_flag, args.err, args.timeout_ns) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + buf * BN + (static_cast<uint32_t>(quad * 32) << 16);
            const bool tma_rows = BN == 256 && args.tma_store != 0 && j.rows >= quad * 32 + 32 &&
                                  !(EPI == EPI_PROJ_ROUTER && j.seg == 1);
            gemm_epilogue_store<BN, EPI>(args, j, row_ok, row, tbase, rs, &tmOut, sOut + quad * 8192, sbuf, tma_rows,
                                         j.a_row0 + quad * 32, lane);
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
