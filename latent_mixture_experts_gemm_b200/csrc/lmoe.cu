// lmoe.cu -- host side of the LatentMoE layer forward: argument checks, the
// workspace plan, TMA descriptors and the launch sequence.  The C ABI is
// declared in include/lmoe.h.
//
// Launch sequence of one forward:
//   router/projection GEMM (tcgen05) -> top-K' + softmax -> counting sort
//   (bitmap, per-expert prefix, offsets + tile lists, scatter/gather) ->
//   up GEMM + activation (tcgen05 grouped; weight streaming for experts with
//   few rows) -> down GEMM (same split) -> combine in the latent width ->
//   up-projection GEMM with the residual add (tcgen05).
// At T <= 32 the projections are split-K weight streams with in-order
// reductions, the router's reduction taking the top-K' too.  The shared
// expert, when present, runs on a second stream of the handle's own.  The
// sequence is captured into a CUDA graph that is launched on the caller's
// stream (forward_graph), or launched there kernel by kernel.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/lmoe.h"
#include "moe_kernels.cuh"
#include "mx.cuh"
#include "nv.cuh"
#include "ep.cuh"
#include "tc_gemm.cuh"
#include "tc_group.cuh"
#include "tc_swap.cuh"

using namespace lmoe;

namespace {

// ------------------------------------------------------------------ driver entry point for TMA descriptors
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool load_encode() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode != nullptr;
}

// bf16 matrix [rows, cols] with row pitch `ld` elements, box = box_rows x 64, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows) {
    if (!load_encode() || rows == 0) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// bf16 matrix [rows, cols] (row pitch `ld` elements) with an unswizzled box of box_rows x box_cols: the output
// blocks the transposed grouped GEMM stages in shared memory row-major.
bool make_map_plain(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_cols,
                    uint32_t box_rows) {
    if (!load_encode() || rows == 0) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld * 2};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Gated expert weights W1 [n_experts][2m][K] bf16 (gate rows, then up rows) as a 5-D tensor
// (K, 16 rows, {gate, up}, m / 16 groups, expert), 128-byte swizzle.  A box of 64 x 16 x 2 x 4 x 1 lands
// as 16 gate rows, their 16 up rows, the next 16 gate rows, ...: 128 rows of 128 bytes.
bool make_map_gated(CUtensorMap* map, const void* base, uint64_t n_experts, uint64_t m, uint64_t K) {
    if (!load_encode() || n_experts == 0 || m % 16 != 0) return false;
    cuuint64_t dims[5] = {K, 16, 2, m / 16, n_experts};
    cuuint64_t strides[4] = {K * 2, m * K * 2, 16 * K * 2, 2 * m * K * 2};
    cuuint32_t box[5] = {64, 16, 2, 4, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides,
                                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Byte matrix [rows, cols] (row pitch `ld` bytes): E4M3 codes (box_cols = 128 with the 128-byte swizzle) or
// block-scale rows (box_cols = 16, no swizzle).
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_cols,
                 uint32_t box_rows, bool swizzle) {
    if (!load_encode() || rows == 0) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE,
                                swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// E2M1 codes [rows, K] packed two per byte in global memory; each load lands as 128 rows x 128 elements with
// every 16 packed elements padded to 16 bytes, the shared-memory form the E2M1 tensor-core operand takes.
bool make_map_e2m1(CUtensorMap* m, const void* base, uint64_t rows, uint64_t K) {
    if (!load_encode() || rows == 0) return false;
    cuuint64_t dims[2] = {K, rows};
    cuuint64_t strides[1] = {K / 2};
    cuuint32_t box[2] = {128, 128};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(base), dims, strides,
                                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// NVFP4 token scale chunks, planar [chunks][rows][16] bytes, seen as 8-byte elements [chunks][2 * rows]: a
// box is 4 chunks x 64 elements, the four 512-byte scale atoms of one 256-element stage (32 rows from the x
// coordinate 2 * first row).  The copy engine's cost grows with the rows of a box: 4 rows of 512 bytes here
// against 128 rows of 16 bytes for a [chunks][rows][16] box of the same bytes.
bool make_map_nv_sf(CUtensorMap* m, const void* base, uint64_t rows, uint64_t chunks) {
    if (!load_encode() || rows == 0) return false;
    cuuint64_t dims[2] = {2 * rows, chunks};
    cuuint64_t strides[1] = {rows * 16};
    cuuint32_t box[2] = {64, 4};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<void*>(base), dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

int n_total(const lmoe_config& c) { return c.n_experts + c.n_zero + c.n_copy + c.n_const; }

bool config_ok(const lmoe_config& c) {
    auto dim_ok = [](int v) { return v >= 64 && v <= 16384 && v % 64 == 0; };
    if (!dim_ok(c.d) || !dim_ok(c.latent) || !dim_ok(c.m)) return false;
    if (c.n_experts < 1 || c.n_zero < 0 || c.n_copy < 0 || c.n_const < 0) return false;
    const int nt = n_total(c);
    if (nt > 1024) return false;
    if (c.top_k < 1 || c.top_k > 32 || c.top_k > nt) return false;
    if (c.max_tokens < 1 || static_cast<long long>(c.max_tokens) * c.top_k > (1LL << 30)) return false;
    if (c.act < 0 || c.act > 2) return false;
    if (c.has_proj != 0 && c.has_proj != 1) return false;
    if (c.latent_router != 0 && c.latent_router != 1) return false;
    if (!c.has_proj && c.latent != c.d) return false;
    if (c.shared_m != 0 && !dim_ok(c.shared_m)) return false;
    if (c.expert_fmt < LMOE_FMT_BF16 || c.expert_fmt > LMOE_FMT_NVFP4) return false;
    // block-scaled experts stream their weights (decode batches) in stages of 128 (MX) or 256 (NVFP4) elements
    const int stage = c.expert_fmt == LMOE_FMT_NVFP4 ? 256 : 128;
    if (c.expert_fmt != LMOE_FMT_BF16 && (c.latent % stage != 0 || c.m % stage != 0)) return false;
    if (c.ep_size < 0 || c.ep_size > 1024) return false;
    if (c.ep_size > 1) {  // expert parallelism: whole local expert sets, bf16 experts
        if (c.n_experts % c.ep_size != 0 || c.ep_rank < 0 || c.ep_rank >= c.ep_size) return false;
        if (c.expert_fmt != LMOE_FMT_BF16) return false;
        const long long n_local = c.n_experts / c.ep_size;
        if (static_cast<long long>(c.ep_size) * c.max_tokens * std::min<long long>(c.top_k, n_local) > (1LL << 30))
            return false;
    } else if (c.ep_rank != 0) {
        return false;
    }
    return true;
}

// Row pitch (bytes) of the block-scale rows of an MXFP8 token operand with K columns: one 16-byte chunk per
// 128-element stage (K is a multiple of 128 for block-scaled experts).
int mx_ld_sf(int K) { return K / 128 * 16; }

// Few-token path (T <= kFewTokenRows): the projections stream their weights
// with split-K on the weight-streaming kernel.
constexpr int kFewTokenRows = 32;
constexpr int kFewTokenMaxSplits = 16;

// Expert-parallel ranks and local FFN experts of a configuration (1 and n_experts without expert parallelism).
int ep_ranks(const lmoe_config& c) { return c.ep_size > 1 ? c.ep_size : 1; }
int n_local_experts(const lmoe_config& c) { return c.n_experts / ep_ranks(c); }

struct Plan {
    size_t hdr, logits, z, zlo, idx, w, bitmap, prefix, counts, offsets, perm, inv, mt_list, pt_list, small_list, rows,
        hbuf, yl,
        partial, hs, s2, partial2, rows4, rows_sf4, h4, h_sf4, rows8, rows_sf, h8, h_sf, xin, xin2, yout, ep_map, ep_src,
        ep_dst, ep_counts,
        ep_offsets, total;
    size_t rows_cap;  // rows of the expert-side buffers: a forward's slots, or the most an experts stage receives
    size_t ep_cap;    // rows an expert-parallel experts stage may receive
    int ld_logits, nwords, mt_max;
};

Plan make_plan(const lmoe_config& c) {
    Plan p{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += round_up(bytes > 0 ? bytes : 1, 256);
        return o;
    };
    const size_t T = c.max_tokens, K = c.top_k, L = c.latent, d = c.d, m = c.m;
    const size_t nt = n_total(c);
    const size_t R = T * K;
    const size_t n_local = n_local_experts(c);
    p.ep_cap = static_cast<size_t>(ep_ranks(c)) * T * std::min(K, n_local);
    p.rows_cap = std::max(R, p.ep_cap);
    const size_t RC = p.rows_cap;
    p.ld_logits = static_cast<int>(round_up(nt, 64));
    p.nwords = static_cast<int>((T + 31) / 32);
    p.mt_max = static_cast<int>((RC + 127) / 128 + c.n_experts);
    p.hdr = take(HDR_WORDS * 4);
    p.logits = take(T * p.ld_logits * 4);
    p.z = c.has_proj ? take(T * L * 2) : 0;
    // latent router: the low bf16 part of the fp32 latent, so the gate reads z at ~16 significant bits
    p.zlo = (c.has_proj && c.latent_router) ? take(T * L * 2) : 0;
    p.idx = take(T * K * 4);
    p.w = take(T * K * 4);
    p.bitmap = take(static_cast<size_t>(p.nwords) * nt * 4);
    p.prefix = take(static_cast<size_t>(p.nwords) * nt * 4);
    p.counts = take(nt * 4);
    p.offsets = take((nt + 1) * 4);
    p.perm = take(R * 4);
    p.inv = take(R * 4);
    p.mt_list = take(static_cast<size_t>(p.mt_max) * 16);
    p.pt_list = take(((RC + 255) / 256 + c.n_experts) * 16);  // CTA-pair tiles: entries of up to 256 rows
    // weight-streaming list: one entry per expert, or (block-scaled experts) one per 32 rows of an expert
    p.small_list = take((static_cast<size_t>(c.n_experts) + RC / SMALL_MAX + 1) * 16);
    p.rows = take(RC * L * 2);  // gathered expert inputs, then (reused) expert outputs
    p.hbuf = take(RC * m * 2);
    p.yl = c.has_proj ? take(T * L * 2) : 0;
    {   // split-K partial sums of the few-token projections: [splits][128-row tiles][32 tokens] fp32
        auto up128 = [](size_t v) { return (v + 127) / 128 * 128; };
        const size_t rows = std::max(up128(L) + up128(nt), std::max(up128(d), up128(nt)));
        p.partial = take(static_cast<size_t>(kFewTokenMaxSplits) * rows * kFewTokenRows * 4);
    }
    if (c.shared_m > 0) {  // shared expert: hidden rows, x + its output, its own split-K partials
        const size_t g = c.act == LMOE_ACT_SWIGLU ? 2 : 1;
        const size_t srows = std::max((g * c.shared_m + 127) / 128 * 128, (d + 127) / 128 * 128);
        p.hs = take(T * static_cast<size_t>(c.shared_m) * 2);
        p.s2 = take(T * d * 2);
        p.partial2 = take(static_cast<size_t>(kFewTokenMaxSplits) * srows * kFewTokenRows * 4);
    }
    if (c.expert_fmt == LMOE_FMT_NVFP4) {  // NVFP4 token operands: packed codes, planar scale chunks
        p.rows4 = take(R * L / 2);
        p.rows_sf4 = take(L / 64 * R * 16);
        p.h4 = take(R * m / 2);
        p.h_sf4 = take(m / 64 * R * 16);
    } else if (c.expert_fmt != LMOE_FMT_BF16) {  // MXFP8 token operands of the expert GEMMs: codes and block scales
        p.rows8 = take(R * L);
        p.rows_sf = take(R * mx_ld_sf(static_cast<int>(L)));
        p.h8 = take(R * m);
        p.h_sf = take(R * mx_ld_sf(static_cast<int>(m)));
    }
    p.xin = take(T * d * 2);
    p.xin2 = take(T * d * 2);  // the host-buffer forward alternates between two input buffers
    p.yout = take(T * d * 2);
    // expert-parallel experts stage: received row -> expert-major row, segment tables, local counts / offsets
    p.ep_map = take(p.ep_cap * 4);
    p.ep_src = take((static_cast<size_t>(c.n_experts) + 1) * 4);
    p.ep_dst = take(static_cast<size_t>(c.n_experts) * 4);
    p.ep_counts = take(n_local * 4);
    p.ep_offsets = take((n_local + 1) * 4);
    p.total = off;
    return p;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

enum Phase : int { PH_ROUTER = 0, PH_TOPK, PH_DISPATCH, PH_UP_TC, PH_UP_STREAM, PH_DOWN_TC, PH_DOWN_STREAM, PH_COMBINE,
                   PH_WUP, PH_SHARED, PH_EP_REGROUP, PH_COUNT };
const char* kPhaseNames[PH_COUNT] = {"router_proj_gemm", "topk_softmax", "dispatch", "expert_up_gemm",
                                     "expert_up_stream", "expert_down_gemm", "expert_down_stream", "combine",
                                     "up_proj_gemm", "shared_expert", "ep_regroup"};

template <int EPI>
bool set_group_attr() {
    return cudaFuncSetAttribute(tc_group_pair_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                GroupCfg::SMEM_BYTES) == cudaSuccess;
}

template <int EPI>
bool set_pair_attr() {
    return cudaFuncSetAttribute(tc_gemm_pair_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                GemmPairCfg::SMEM_BYTES) == cudaSuccess;
}

template <int BN, int EPI>
bool set_smem_attr() {
    return cudaFuncSetAttribute(tc_gemm_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                GemmCfg<BN>::SMEM_BYTES) == cudaSuccess;
}

// Kernel launch with programmatic dependent launch: the kernel may be placed
// while its predecessor in the stream drains; every kernel of the layer waits
// for its predecessor first thing (pdl_begin), so results are unchanged.
bool g_use_pdl = true;

// The same for a kernel of CTA pairs: clusters of 2 along x (grid.x even).
template <typename... P, typename... A>
void launch_pairs(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, A&&... args) {
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = g_use_pdl ? 2 : 1;
    cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

template <typename... P, typename... A>
void launch(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, A&&... args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = g_use_pdl ? 1 : 0;
    cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

template <int NT, int EPI>
bool set_swap_attr() {
    return cudaFuncSetAttribute(tc_swap_kernel<NT, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SwapCfg<NT, EPI>::SMEM_BYTES) == cudaSuccess;
}

template <int EPI, bool W4, bool QOUT>
bool set_mx_attr() {
    return cudaFuncSetAttribute(tc_swap_mx_kernel<EPI, W4, QOUT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                MxCfg<EPI, W4>::SMEM_BYTES) == cudaSuccess;
}

template <int EPI, bool QOUT>
bool set_nv_attr() {
    return cudaFuncSetAttribute(tc_swap_nv_kernel<EPI, QOUT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                NvCfg<EPI>::SMEM_BYTES) == cudaSuccess;
}

bool set_all_smem_attrs() {
    bool ok = true;
    ok &= set_nv_attr<EPI_BF16, true>();
    ok &= set_nv_attr<EPI_RELU2, true>();
    ok &= set_nv_attr<EPI_SWIGLU, true>();
    ok &= set_nv_attr<EPI_BF16, false>();
    ok &= set_group_attr<EPI_BF16>();
    ok &= set_group_attr<EPI_RELU2>();
    ok &= set_group_attr<EPI_SWIGLU>();
    ok &= set_pair_attr<EPI_BF16>();
    ok &= set_pair_attr<EPI_RELU2>();
    ok &= set_pair_attr<EPI_SWIGLU>();
    ok &= set_pair_attr<EPI_RESID>();
    ok &= set_pair_attr<EPI_PROJ_ROUTER>();
    ok &= set_mx_attr<EPI_BF16, false, true>();
    ok &= set_mx_attr<EPI_RELU2, false, true>();
    ok &= set_mx_attr<EPI_SWIGLU, false, true>();
    ok &= set_mx_attr<EPI_BF16, false, false>();
    ok &= set_mx_attr<EPI_BF16, true, true>();
    ok &= set_mx_attr<EPI_RELU2, true, true>();
    ok &= set_mx_attr<EPI_SWIGLU, true, true>();
    ok &= set_mx_attr<EPI_BF16, true, false>();
    ok &= cudaFuncSetAttribute(dispatch_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (2 * SMALL_BATCH_WORDS * 1024 + 1024) * 4) == cudaSuccess;
    ok &= set_swap_attr<16, EPI_BF16>();
    ok &= set_swap_attr<16, EPI_RELU2>();
    ok &= set_swap_attr<16, EPI_SWIGLU>();
    ok &= set_swap_attr<32, EPI_BF16>();
    ok &= set_swap_attr<32, EPI_RELU2>();
    ok &= set_swap_attr<32, EPI_SWIGLU>();
    ok &= set_smem_attr<64, EPI_BF16>();
    ok &= set_smem_attr<256, EPI_BF16>();
    ok &= set_smem_attr<64, EPI_RESID>();
    ok &= set_smem_attr<256, EPI_RESID>();
    ok &= set_smem_attr<64, EPI_PROJ_ROUTER>();
    ok &= set_smem_attr<256, EPI_PROJ_ROUTER>();
    ok &= set_smem_attr<64, EPI_RELU2>();
    ok &= set_smem_attr<64, EPI_SWIGLU>();
    ok &= set_smem_attr<256, EPI_RELU2>();
    ok &= set_smem_attr<256, EPI_SWIGLU>();
    // the per-token scatter holds one feature row (at most 16384 bf16) per warp
    ok &= cudaFuncSetAttribute(dispatch_scatter_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SCATTER_WARPS * 16384 * 2) == cudaSuccess;
    return ok;
}

// `x2`: the token operand of the k-blocks past args.k_wrap (nullptr: none, x stands in).
template <int NT, int EPI>
void launch_swap(const CUtensorMap& w, const CUtensorMap& x, const CUtensorMap& w2, const SwapArgs& args, int grid,
                 cudaStream_t s, const CUtensorMap* x2 = nullptr) {
    launch(tc_swap_kernel<NT, EPI>, grid, 192, SwapCfg<NT, EPI>::SMEM_BYTES, s, w, x, w2, x2 != nullptr ? *x2 : x,
           args);
}

// Weight-streaming launch for the experts of the small list, dispatched on the token tile and epilogue.
void launch_stream(int nt, int epi, const CUtensorMap& w, const CUtensorMap& x16, const CUtensorMap& x32,
                   const SwapArgs& a, int grid, cudaStream_t s) {
    if (nt <= 16) {
        if (epi == EPI_RELU2) launch_swap<16, EPI_RELU2>(w, x16, w, a, grid, s);
        else if (epi == EPI_SWIGLU) launch_swap<16, EPI_SWIGLU>(w, x16, w, a, grid, s);
        else launch_swap<16, EPI_BF16>(w, x16, w, a, grid, s);
    } else {
        if (epi == EPI_RELU2) launch_swap<32, EPI_RELU2>(w, x32, w, a, grid, s);
        else if (epi == EPI_SWIGLU) launch_swap<32, EPI_SWIGLU>(w, x32, w, a, grid, s);
        else launch_swap<32, EPI_BF16>(w, x32, w, a, grid, s);
    }
}

// Few-token projection: split-K weight streaming into fp32 partials, then the
// in-order reduction with its epilogue.  Returns the number of launches.
struct FewTokenGemm {
    const CUtensorMap* w;   // first weight segment (128-row boxes)
    const CUtensorMap* w2;  // second weight segment (or the same map)
    const CUtensorMap* x16;
    const CUtensorMap* x32;
    int rows0, rows1;       // weight rows of the two segments (rows1 may be 0)
    int K;
    __nv_bfloat16* out0;
    int ld0;
    float* out1;
    int ld1;
    const __nv_bfloat16* resid;
    int ld_resid;
    int act = EPI_BF16;     // activation of segment 0 (EPI_RELU2 / EPI_SWIGLU: gate rows first, then up rows)
    int out_cols0 = -1;     // output columns of segment 0 (default rows0; rows0 / 2 when gated)
    __nv_bfloat16* out0_lo = nullptr;  // segment 0 without activation: also the low part bf16(v - bf16(v))
    // two-part token operand: K = 2 * k_wrap, the k-blocks past k_wrap read x16b / x32b and the weights again
    int k_wrap = 0;
    const CUtensorMap* x16b = nullptr;
    const CUtensorMap* x32b = nullptr;
    // router: with topk_idx set, segment 1 holds the router logits, and the reduction also selects each
    // token's top-K' (bias added) and writes ids and renormalised weights
    const float* bias = nullptr;
    int topk = 0;
    int32_t* topk_idx = nullptr;
    float* topk_w = nullptr;
};

template <int NT>
void launch_few_token_reduce(const FewTokenGemm& g, int T, const float* partial, int part_rows, int splits, int t0,
                             cudaStream_t s) {
    const int n0 = g.out_cols0 >= 0 ? g.out_cols0 : g.rows0;
    const long outs = static_cast<long>(n0 + g.rows1) * T;
    const unsigned rgrid = static_cast<unsigned>((outs + 255) / 256);
#define LMOE_REDUCE(A)                                                                                           \
    launch(swap_reduce_kernel<NT, A>, rgrid, 256, 0, s, partial, part_rows, splits, T, n0, g.rows1, t0 * 128, n0, \
           g.out0, g.ld0, g.out1, g.ld1, g.resid, g.ld_resid, A == EPI_BF16 ? g.out0_lo : nullptr)
    if (g.act == EPI_RELU2) LMOE_REDUCE(EPI_RELU2);
    else if (g.act == EPI_SWIGLU) LMOE_REDUCE(EPI_SWIGLU);
    else LMOE_REDUCE(EPI_BF16);
#undef LMOE_REDUCE
}

// The router's reduction with the top-K' selection: one block per token (segment 1 = the logits, no
// activation on segment 0).
template <int NT>
void launch_router_reduce_topk(const FewTokenGemm& g, int T, const float* partial, int part_rows, int splits, int t0,
                               cudaStream_t s) {
    const int n1 = g.rows1, npl = (n1 + 31) / 32;
    const size_t smem = static_cast<size_t>(n1) * 4;
    // T routing blocks, then the z columns at one element per thread
    const unsigned grid = static_cast<unsigned>(T + (static_cast<long>(g.rows0) * T + 511) / 512);
#define LMOE_RTOPK(N)                                                                                             \
    launch(router_reduce_topk_kernel<NT, N>, grid, 512, smem, s, partial, part_rows, splits, T, g.rows0, n1,      \
           t0 * 128, g.out0, g.ld0, g.out1, g.ld1, g.bias, g.topk, g.topk_idx, g.topk_w)
    if (npl <= 1) LMOE_RTOPK(1);
    else if (npl <= 2) LMOE_RTOPK(2);
    else if (npl <= 4) LMOE_RTOPK(4);
    else if (npl <= 8) LMOE_RTOPK(8);
    else if (npl <= 16) LMOE_RTOPK(16);
    else LMOE_RTOPK(32);
#undef LMOE_RTOPK
}

int launch_few_token(const FewTokenGemm& g, int T, float* partial, int max_splits, int num_sms, int* err,
                     unsigned long long timeout_ns, cudaStream_t s) {
    const int t0 = (g.rows0 + 127) / 128, t1 = (g.rows1 + 127) / 128;
    const int nkb = g.K / 64;
    // Each (weight tile, K split) unit streams a 512-deep slice of K, 128 KB of weights, and there is at
    // most one unit per SM.  Longer units beat one unit per SM: each split costs a CTA's fixed set-up and
    // adds a block of partial sums to the in-order reduction.
    int splits = std::min((num_sms + t0 + t1 - 1) / (t0 + t1), (nkb + 7) / 8);
    splits = std::max(1, std::min(splits, std::min(max_splits, nkb)));
    SwapArgs a{};
    a.K = g.K;
    a.n_wtiles = t0 + t1;
    a.n_wtiles0 = t0;
    a.k_splits = splits;
    a.list = nullptr;
    a.dense_rows = T;
    a.partial = partial;
    a.part_rows = (t0 + t1) * 128;
    a.err = err;
    a.timeout_ns = timeout_ns;
    a.k_wrap = g.k_wrap;
    const int grid = std::min(num_sms, (t0 + t1) * splits);
    if (T <= 16) {
        launch_swap<16, EPI_BF16>(*g.w, *g.x16, *g.w2, a, grid, s, g.k_wrap > 0 ? g.x16b : nullptr);
        if (g.topk_idx != nullptr) launch_router_reduce_topk<16>(g, T, partial, a.part_rows, splits, t0, s);
        else launch_few_token_reduce<16>(g, T, partial, a.part_rows, splits, t0, s);
    } else {
        launch_swap<32, EPI_BF16>(*g.w, *g.x32, *g.w2, a, grid, s, g.k_wrap > 0 ? g.x32b : nullptr);
        if (g.topk_idx != nullptr) launch_router_reduce_topk<32>(g, T, partial, a.part_rows, splits, t0, s);
        else launch_few_token_reduce<32>(g, T, partial, a.part_rows, splits, t0, s);
    }
    return 2;
}

// `out` (optional): TMA map of the bf16 output (box 32 rows x 64 columns, 128-byte swizzle); the epilogue
// then stores whole 32-row blocks with TMA (BN = 256).  Without it every thread stores its own row.
// `a2` (optional): the A operand of the k-blocks past args.k_wrap.
template <int BN, int EPI>
void launch_gemm(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& b2, const GemmArgs& args, int grid,
                 cudaStream_t s, const CUtensorMap* out = nullptr, const CUtensorMap* a2 = nullptr) {
    GemmArgs g = args;
    g.tma_store = (out != nullptr && BN == 256) ? 1 : 0;
    launch(tc_gemm_kernel<BN, EPI>, grid, 192, GemmCfg<BN>::SMEM_BYTES, s, a, b, b2, out != nullptr ? *out : a,
           a2 != nullptr ? *a2 : a, g);
}

// CTA-pair GEMM: `pair_tiles` (or, for a device-built list, an upper bound) pair tiles on up to num_sms / 2 pairs.
template <int EPI>
void launch_gemm_pair(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& b2, const GemmArgs& args,
                      int pair_tiles, int num_sms, cudaStream_t s, const CUtensorMap* out = nullptr,
                      const CUtensorMap* a2 = nullptr) {
    const int pairs = std::max(1, std::min(num_sms / 2, pair_tiles));
    GemmArgs g = args;
    g.tma_store = out != nullptr ? 1 : 0;
    launch_pairs(tc_gemm_pair_kernel<EPI>, 2 * pairs, 192, GemmPairCfg::SMEM_BYTES, s, a, b, b2,
                 out != nullptr ? *out : a, a2 != nullptr ? *a2 : a, g);
}

// Grouped expert GEMM on CTA pairs (computed transposed): one pair per two SMs, persistent.
// x32 / x64 / x128: the token rows (K-major, 128-byte swizzle) in boxes of 32, 64 and 128 rows.
template <int EPI>
void launch_group(const CUtensorMap& w, const CUtensorMap& x32, const CUtensorMap& x64, const CUtensorMap& x128,
                  const CUtensorMap& out, const GroupArgs& a, int num_sms, cudaStream_t s) {
    launch_pairs(tc_group_pair_kernel<EPI>, 2 * (num_sms / 2), GroupCfg::THREADS, GroupCfg::SMEM_BYTES, s, w, x32, x64,
                 x128, out, a);
}

template <int EPI, bool W4, bool QOUT>
void launch_mx(const CUtensorMap& w, const CUtensorMap& x, const CUtensorMap& xsf, const MxArgs& a, int grid,
               cudaStream_t s) {
    launch(tc_swap_mx_kernel<EPI, W4, QOUT>, grid, 192, MxCfg<EPI, W4>::SMEM_BYTES, s, w, x, xsf, a);
}

// Block-scaled expert phase: the up GEMM (activation, MXFP8 re-encoding) or the down GEMM (bf16 out).
template <int EPI, bool QOUT>
void launch_nv(const CUtensorMap& w, const CUtensorMap& x, const CUtensorMap& xsf, const NvArgs& a, int grid,
               cudaStream_t s) {
    launch(tc_swap_nv_kernel<EPI, QOUT>, grid, NvCfg<EPI>::THREADS, NvCfg<EPI>::SMEM_BYTES, s, w, x, xsf, a);
}
void launch_nv_phase(bool up, int epi, const CUtensorMap& w, const CUtensorMap& x, const CUtensorMap& xsf,
                     const NvArgs& a, int grid, cudaStream_t s) {
    if (!up) launch_nv<EPI_BF16, false>(w, x, xsf, a, grid, s);
    else if (epi == EPI_RELU2) launch_nv<EPI_RELU2, true>(w, x, xsf, a, grid, s);
    else if (epi == EPI_SWIGLU) launch_nv<EPI_SWIGLU, true>(w, x, xsf, a, grid, s);
    else launch_nv<EPI_BF16, true>(w, x, xsf, a, grid, s);
}
void launch_mx_phase(bool up, int epi, bool w4, const CUtensorMap& w, const CUtensorMap& x, const CUtensorMap& xsf,
                     const MxArgs& a, int grid, cudaStream_t s) {
    if (!up) {
        if (w4) launch_mx<EPI_BF16, true, false>(w, x, xsf, a, grid, s);
        else launch_mx<EPI_BF16, false, false>(w, x, xsf, a, grid, s);
    } else if (epi == EPI_RELU2) {
        if (w4) launch_mx<EPI_RELU2, true, true>(w, x, xsf, a, grid, s);
        else launch_mx<EPI_RELU2, false, true>(w, x, xsf, a, grid, s);
    } else if (epi == EPI_SWIGLU) {
        if (w4) launch_mx<EPI_SWIGLU, true, true>(w, x, xsf, a, grid, s);
        else launch_mx<EPI_SWIGLU, false, true>(w, x, xsf, a, grid, s);
    } else {
        if (w4) launch_mx<EPI_BF16, true, true>(w, x, xsf, a, grid, s);
        else launch_mx<EPI_BF16, false, true>(w, x, xsf, a, grid, s);
    }
}

}  // namespace

// ====================================================================== handle
struct lmoe_handle {
    lmoe_config c{};
    lmoe_weights w{};
    uint8_t* ws = nullptr;
    Plan p{};
    int n_tot = 0, g = 1, num_sms = 148, small_max = 16, device = 0;
    int n_local = 1;      // FFN experts whose weights this handle holds
    int last_small = 16;  // threshold the last forward used
    // expert-parallel forward in progress: the dispatch's x and T (ep_T < 0: none)
    const void* ep_x = nullptr;
    int ep_T = -1;
    int64_t ep_block_rows = 0;  // the forward in progress exchanges rank blocks of this many rows (0: packed)
    bool stats_ep = false;  // the header's row / tile counts are those of the last experts stage
    unsigned long long timeout_ns = 1000000000ull;
    // weight descriptors: router/projection operands for both column tiles, expert weights, workspace operands
    CUtensorMap wdown64{}, wdown256{}, wr64{}, wr256{}, wup64{}, wup256{}, w1{}, w2{};
    CUtensorMap a_rows{}, a_h{}, a_yl{}, a_z{};
    // weight-streaming operands: 128-row weight tiles, 16- and 32-row token tiles
    CUtensorMap w1s{}, w2s{}, rows16{}, rows32{}, h16{}, h32{};
    // few-token projections: 128-row weight tiles and 16/32-row token tiles of z and yl
    CUtensorMap wdown128{}, wr128{}, wup128{}, z16{}, z32{}, yl16{}, yl32{};
    // latent router: the latent's low part as the second A operand (128-row tiles) and token operand (16/32)
    CUtensorMap a_zlo{}, zlo16{}, zlo32{};
    // shared expert: weights for 64/256-column tiles (gated: half-tile boxes), 128-row weight tiles,
    // its hidden rows as the A operand (128-row tiles) and as 16/32-row token tiles
    CUtensorMap ws1_64{}, ws1_256{}, ws2_64{}, ws2_256{}, ws1_128{}, ws2_128{}, a_hs{}, hs16{}, hs32{};
    // block-scaled experts: weight codes (128 x 128 boxes) and the MXFP8 token operands with their scales
    CUtensorMap w1q{}, w2q{}, rows8{}, rows_sf{}, h8{}, h_sf{};
    // NVFP4 experts: packed weight codes (128 x 128-byte boxes), token codes (32 x 128-byte boxes) and the
    // token scale chunks (4 rows of 512 bytes: one stage's four atoms)
    CUtensorMap w1n{}, w2n{}, rows4{}, rows_sf4{}, h4{}, h_sf4{};
    // TMA store maps of bf16 GEMM outputs (32-row x 64-column boxes): hidden rows, expert outputs, z
    CUtensorMap o_h{}, o_rows{}, o_z{};
    // grouped expert GEMMs on CTA pairs (transposed): gated W1 as 16-row gate / up groups, unswizzled output blocks of
    // 32 rows x 32 (x 16 for gated) columns of the hidden rows and of the expert outputs
    CUtensorMap w1g16{}, og_h{}, og_rows{}, rows64{}, h64{};
    bool group_pair_ok = false;  // the shapes allow it: m (gated: m / 2 per pair tile) and latent in 256-row tiles
    int group_pair = 0;          // 1: grouped expert GEMMs on CTA pairs; 0 (default): single-CTA 128-row tiles
    cudaStream_t side = nullptr;     // the shared expert runs here, concurrently with the routed path
    // lmoe_forward_host: the input copy runs on `hcopy` into one of two input buffers, so that the copy of
    // one call overlaps the forward of the one before; ev_in[b] marks buffer b's copy done, ev_used[b] the
    // forward that read it done
    cudaStream_t hcopy = nullptr;
    cudaEvent_t ev_in[2] = {nullptr, nullptr}, ev_used[2] = {nullptr, nullptr};
    uint64_t host_calls = 0;
    // Forwards launched as a CUDA graph: each call captures its launches on `cap` and replays them on the
    // caller's stream from an executable graph, updated in place.  A few executable graphs are kept, one per
    // launch sequence (token counts that change the kernels used), least recently used first out.
    struct GraphExec {
        std::vector<const void*> sig;  // node kinds and kernel functions, in the capture's order
        cudaGraphExec_t exec = nullptr;
        uint64_t used = 0;
    };
    cudaStream_t cap = nullptr;
    std::vector<GraphExec> graphs;
    uint64_t graph_tick = 0;
    int use_graph = 1;
    cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
    // profiling
    bool prof = false;
    int prof_max = 0, prof_n = 0;
    std::vector<cudaEvent_t> ev;
    std::vector<int> launches;
    template <typename T>
    T* at(size_t off) const { return reinterpret_cast<T*>(ws + off); }
};

namespace {

struct PhaseScope {
    lmoe_handle* h;
    int ph;
    cudaStream_t s;
    int n_launch;
    bool on;
    PhaseScope(lmoe_handle* h_, int ph_, cudaStream_t s_, int n) : h(h_), ph(ph_), s(s_), n_launch(n) {
        on = h->prof && h->prof_n < h->prof_max;
        if (on) cudaEventRecord(h->ev[(static_cast<size_t>(h->prof_n) * PH_COUNT + ph) * 2], s);
    }
    ~PhaseScope() {
        if (on) {
            cudaEventRecord(h->ev[(static_cast<size_t>(h->prof_n) * PH_COUNT + ph) * 2 + 1], s);
            h->launches[static_cast<size_t>(h->prof_n) * PH_COUNT + ph] = n_launch;
        }
    }
};

void free_events(lmoe_handle* h) {
    for (cudaEvent_t e : h->ev)
        if (e) cudaEventDestroy(e);
    h->ev.clear();
    h->launches.clear();
    h->prof_max = h->prof_n = 0;
}

// Shared expert (forked to the side stream), router (+ W_down), top-K' and the
// counting sort by expert.  The feature rows of slots routed to FFN experts are
// gathered in sorted order to `rows_dst` (ld = latent), or encoded as the MXFP8
// token operand for block-scaled experts; `small` shapes the tile lists.
int run_front(lmoe_handle* h, const void* x, int T, cudaStream_t s, __nv_bfloat16* rows_dst, int small) {
    const lmoe_config& c = h->c;
    const Plan& p = h->p;
    const int K = c.top_k, L = c.latent, d = c.d, nt = h->n_tot;
    const bool proj = c.has_proj != 0;
    const bool mx = c.expert_fmt != LMOE_FMT_BF16;
    int* hdr = h->at<int>(p.hdr);
    float* logits = h->at<float>(p.logits);
    __nv_bfloat16* z = proj ? h->at<__nv_bfloat16>(p.z) : nullptr;
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
    const __nv_bfloat16* feat = proj ? z : xb;  // what the experts read (latent z, or x for the standard MoE)
    int32_t* idx = h->at<int32_t>(p.idx);
    float* wts = h->at<float>(p.w);
    int4* mt_list = h->at<int4>(p.mt_list);
    int4* small_list = h->at<int4>(p.small_list);
    const int nwords = (T + 31) / 32;
    int* counts = h->at<int>(p.counts);
    int* offsets = h->at<int>(p.offsets);
    int32_t* perm = h->at<int32_t>(p.perm);
    int32_t* inv = h->at<int32_t>(p.inv);
    const long slots = static_cast<long>(T) * K;
    const int npl = (nt + 31) / 32;
    const float* bias = h->w.router_bias;

    CUtensorMap a_x;
    if (!make_map(&a_x, x, T, d, d, 128)) return LMOE_ERR_CUDA;
    const int m_tiles = (T + 127) / 128;

    GemmArgs base{};
    base.err = hdr + HDR_ERR;
    base.timeout_ns = h->timeout_ns;

    // ---------------------------------------------------------------- shared expert (side stream)
    // s2 = x + Ws2 act(Ws1 x) runs concurrently with the routed path; the up-projection
    // (or, for the standard MoE, the combine) waits for it and adds s2 instead of x.
    if (c.shared_m > 0) {
        const int ms = c.shared_m, srows = h->g * ms;
        __nv_bfloat16* hs = h->at<__nv_bfloat16>(p.hs);
        __nv_bfloat16* s2 = h->at<__nv_bfloat16>(p.s2);
        const int epi = c.act == LMOE_ACT_SWIGLU ? EPI_SWIGLU : (c.act == LMOE_ACT_RELU2 ? EPI_RELU2 : EPI_BF16);
        if (cudaEventRecord(h->ev_fork, s) != cudaSuccess || cudaStreamWaitEvent(h->side, h->ev_fork, 0) != cudaSuccess)
            return LMOE_ERR_CUDA;
        {
            PhaseScope ps(h, PH_SHARED, h->side, T <= kFewTokenRows ? 4 : 2);
            if (T <= kFewTokenRows) {
                CUtensorMap x16, x32;
                if (!make_map(&x16, x, T, d, d, 16) || !make_map(&x32, x, T, d, d, 32)) return LMOE_ERR_CUDA;
                float* part2 = h->at<float>(p.partial2);
                FewTokenGemm up{&h->ws1_128, &h->ws1_128, &x16, &x32, srows, 0, d, hs, ms, nullptr, 0, nullptr, 0};
                up.act = epi;
                up.out_cols0 = ms;
                launch_few_token(up, T, part2, kFewTokenMaxSplits, h->num_sms, hdr + HDR_ERR, h->timeout_ns, h->side);
                FewTokenGemm dn{&h->ws2_128, &h->ws2_128, &h->hs16, &h->hs32, d, 0, ms, s2, d, nullptr, 0, xb, d};
                launch_few_token(dn, T, part2, kFewTokenMaxSplits, h->num_sms, hdr + HDR_ERR, h->timeout_ns, h->side);
            } else {
                GemmArgs a = base;
                a.M = T;
                a.K = d;
                a.N0 = ms;
                a.out0 = hs;
                a.ld0 = ms;
                a.up_offset = ms;
                const bool big_up = m_tiles * ((ms + (epi == EPI_SWIGLU ? 127 : 255)) / (epi == EPI_SWIGLU ? 128 : 256)) >=
                                    h->num_sms;
                if (big_up) {
                    a.n_tiles = epi == EPI_SWIGLU ? (ms + 127) / 128 : (ms + 255) / 256;
                    const int grid = std::min(h->num_sms, m_tiles * a.n_tiles);
                    if (epi == EPI_SWIGLU) launch_gemm<256, EPI_SWIGLU>(a_x, h->ws1_256, h->ws1_256, a, grid, h->side);
                    else if (epi == EPI_RELU2) launch_gemm<256, EPI_RELU2>(a_x, h->ws1_256, h->ws1_256, a, grid, h->side);
                    else launch_gemm<256, EPI_BF16>(a_x, h->ws1_256, h->ws1_256, a, grid, h->side);
                } else {
                    a.n_tiles = epi == EPI_SWIGLU ? (ms + 31) / 32 : (ms + 63) / 64;
                    const int grid = std::min(h->num_sms, m_tiles * a.n_tiles);
                    if (epi == EPI_SWIGLU) launch_gemm<64, EPI_SWIGLU>(a_x, h->ws1_64, h->ws1_64, a, grid, h->side);
                    else if (epi == EPI_RELU2) launch_gemm<64, EPI_RELU2>(a_x, h->ws1_64, h->ws1_64, a, grid, h->side);
                    else launch_gemm<64, EPI_BF16>(a_x, h->ws1_64, h->ws1_64, a, grid, h->side);
                }
                GemmArgs b = base;
                b.M = T;
                b.K = ms;
                b.N0 = d;
                b.out0 = s2;
                b.ld0 = d;
                b.resid = xb;
                b.ld_resid = d;
                if (m_tiles * ((d + 255) / 256) >= h->num_sms) {
                    b.n_tiles = (d + 255) / 256;
                    launch_gemm<256, EPI_RESID>(h->a_hs, h->ws2_256, h->ws2_256, b, std::min(h->num_sms, m_tiles * b.n_tiles),
                                                h->side);
                } else {
                    b.n_tiles = (d + 63) / 64;
                    launch_gemm<64, EPI_RESID>(h->a_hs, h->ws2_64, h->ws2_64, b, std::min(h->num_sms, m_tiles * b.n_tiles),
                                               h->side);
                }
            }
        }
        if (cudaEventRecord(h->ev_join, h->side) != cudaSuccess) return LMOE_ERR_CUDA;
    }

    // ---------------------------------------------------------------- router (+ W_down)
    if (T <= kFewTokenRows) {
        // few tokens: split-K weight streaming (weights as the 128-row operand), then the in-order reduction,
        // which also takes each token's top-K' and softmax from its logits (router_reduce_topk_kernel)
        CUtensorMap x16, x32;
        if (!make_map(&x16, x, T, d, d, 16) || !make_map(&x32, x, T, d, d, 32)) return LMOE_ERR_CUDA;
        float* part = h->at<float>(p.partial);
        const bool fused = proj && !c.latent_router;
        const int n_launch = (proj && c.latent_router) ? 4 : 2;
        PhaseScope ps(h, PH_ROUTER, s, n_launch);
        auto with_topk = [&](FewTokenGemm& r) {
            r.bias = bias;
            r.topk = K;
            r.topk_idx = idx;
            r.topk_w = wts;
        };
        if (proj && c.latent_router) {
            // z = hi + lo from the fp32 sum; the gate multiplies both parts (K = 2L, its weights streamed
            // twice), so it reads the latent at ~16 significant bits instead of bf16's 8
            FewTokenGemm g{&h->wdown128, &h->wdown128, &x16, &x32, L, 0, d, z, L, nullptr, 0, nullptr, 0};
            g.out0_lo = h->at<__nv_bfloat16>(p.zlo);
            launch_few_token(g, T, part, kFewTokenMaxSplits, h->num_sms, hdr + HDR_ERR, h->timeout_ns, s);
            FewTokenGemm r{&h->wr128, &h->wr128, &h->z16, &h->z32, 0, nt, 2 * L, nullptr, 0, logits, p.ld_logits,
                           nullptr, 0};
            r.k_wrap = L;
            r.x16b = &h->zlo16;
            r.x32b = &h->zlo32;
            with_topk(r);
            launch_few_token(r, T, part, kFewTokenMaxSplits, h->num_sms, hdr + HDR_ERR, h->timeout_ns, s);
        } else if (fused) {
            FewTokenGemm g{&h->wdown128, &h->wr128, &x16, &x32, L, nt, d, z, L, logits, p.ld_logits, nullptr, 0};
            with_topk(g);
            launch_few_token(g, T, part, kFewTokenMaxSplits, h->num_sms, hdr + HDR_ERR, h->timeout_ns, s);
        } else {
            FewTokenGemm r{&h->wr128, &h->wr128, &x16, &x32, 0, nt, d, nullptr, 0, logits, p.ld_logits, nullptr, 0};
            with_topk(r);
            launch_few_token(r, T, part, kFewTokenMaxSplits, h->num_sms, hdr + HDR_ERR, h->timeout_ns, s);
        }
    } else {
        {
            const bool fused = proj && !c.latent_router;
            const int n256 = (fused ? (L + 255) / 256 : 0) + (nt + 255) / 256;
            const bool big = m_tiles * n256 >= h->num_sms;
            const int n_gemm = (proj && c.latent_router) ? 2 : 1;
            PhaseScope ps(h, PH_ROUTER, s, n_gemm);
            if (proj && c.latent_router) {
                // z (bf16) and its low part zlo = bf16(z32 - z) from the fp32 accumulator
                GemmArgs a = base;
                a.M = T;
                a.K = d;
                a.N0 = L;
                a.out0 = z;
                a.ld0 = L;
                a.out_lo = h->at<__nv_bfloat16>(p.zlo);
                if (big) {
                    a.n_tiles = (L + 255) / 256;
                    launch_gemm<256, EPI_BF16>(a_x, h->wdown256, h->wdown256, a, std::min(h->num_sms, m_tiles * a.n_tiles), s);
                } else {
                    a.n_tiles = (L + 63) / 64;
                    launch_gemm<64, EPI_BF16>(a_x, h->wdown64, h->wdown64, a, std::min(h->num_sms, m_tiles * a.n_tiles), s);
                }
            }
            GemmArgs a = base;
            a.M = T;
            a.K = c.latent_router ? L : d;
            if (proj && c.latent_router) {  // the gate reads z + zlo: K = 2L, the router weights read twice
                a.K = 2 * L;
                a.k_wrap = L;
            }
            a.N0 = fused ? L : 0;
            a.N1 = nt;
            a.out0 = z;
            a.ld0 = L;
            a.out1 = logits;
            a.ld1 = p.ld_logits;
            const CUtensorMap& A = (proj && c.latent_router) ? h->a_z : a_x;
            if (big) {
                a.n_tiles0 = fused ? (L + 255) / 256 : 0;
                a.n_tiles = a.n_tiles0 + (nt + 255) / 256;
                launch_gemm_pair<EPI_PROJ_ROUTER>(A, fused ? h->wdown128 : h->wr128, h->wr128, a,
                                                  (T + 255) / 256 * a.n_tiles, h->num_sms, s, fused ? &h->o_z : nullptr,
                                                  a.k_wrap > 0 ? &h->a_zlo : nullptr);
            } else {
                a.n_tiles0 = fused ? (L + 63) / 64 : 0;
                a.n_tiles = a.n_tiles0 + (nt + 63) / 64;
                launch_gemm<64, EPI_PROJ_ROUTER>(A, fused ? h->wdown64 : h->wr64, h->wr64, a,
                                                 std::min(h->num_sms, m_tiles * a.n_tiles), s, nullptr,
                                                 a.k_wrap > 0 ? &h->a_zlo : nullptr);
            }
        }
    }
    // ---------------------------------------------------------------- top-K' + softmax (T > 32: its own kernel)
    if (T > kFewTokenRows) {
        PhaseScope ps(h, PH_TOPK, s, 1);
        const dim3 grid((T + 3) / 4), block(128);  // one warp per token, 4 per block (few tokens: more SMs)
#define LMOE_TOPK(N) launch(topk_softmax_kernel<N>, grid, block, 0, s, logits, p.ld_logits, bias, T, nt, K, idx, wts)
        if (npl <= 1) LMOE_TOPK(1);
        else if (npl <= 2) LMOE_TOPK(2);
        else if (npl <= 4) LMOE_TOPK(4);
        else if (npl <= 8) LMOE_TOPK(8);
        else if (npl <= 16) LMOE_TOPK(16);
        else LMOE_TOPK(32);
#undef LMOE_TOPK
    }
    // ---------------------------------------------------------------- counting sort by expert (+ row gather)
    if (nwords <= SMALL_BATCH_WORDS) {
        PhaseScope ps(h, PH_DISPATCH, s, 2);
        const size_t sm = (static_cast<size_t>(2 * nwords) * nt + nt) * 4;
        launch(dispatch_small_kernel, 1, 1024, sm, s, idx, T, K, nt, c.n_experts, small, counts, offsets, mt_list,
               small_list, h->at<int4>(p.pt_list), perm, inv, hdr);
        if (c.expert_fmt == LMOE_FMT_NVFP4)
            launch(nv_gather_kernel, static_cast<unsigned>((slots + 7) / 8), 256, 0, s, idx, inv, T, K, c.n_experts,
                   feat, L, L, h->at<uint8_t>(p.rows4), h->at<uint8_t>(p.rows_sf4), static_cast<int>(c.max_tokens) * K);
        else if (mx)
            launch(mx_gather_kernel, static_cast<unsigned>((slots + 7) / 8), 256, 0, s, idx, inv, T, K, c.n_experts,
                   feat, L, L, h->at<uint8_t>(p.rows8), L, h->at<uint8_t>(p.rows_sf), mx_ld_sf(L));
        else
            launch(dispatch_gather_kernel, static_cast<unsigned>((slots + 7) / 8), 256, 0, s, idx, inv, T, K,
                   c.n_experts, feat, L, L, rows_dst, L);
    } else {
        PhaseScope ps(h, PH_DISPATCH, s, mx ? 5 : 4);
        uint32_t* bitmap = h->at<uint32_t>(p.bitmap);
        uint32_t* prefix = h->at<uint32_t>(p.prefix);
        launch(dispatch_bitmap_kernel, (nwords + 7) / 8, 256, 8 * nt * 4, s, idx, T, K, nt, bitmap, hdr);
        launch(dispatch_expert_scan_kernel, (nt + 7) / 8, 256, 0, s, bitmap, T, nt, prefix, counts);
        launch(dispatch_offsets_kernel, 1, 1024, 0, s, counts, nt, c.n_experts, small, offsets, mt_list, small_list,
               h->at<int4>(p.pt_list), hdr);
        // block-scaled experts: the scatter only places the slots (no bf16 row copy); the gather encodes the rows.
        // With many slots per token the row is read once and written by bulk copies (measured: Nemotron-like
        // prefill 111-117 -> 103 us, Kimi-like 76 -> 68 us); with few (top-6 of the standard MoE, 8 KB rows) the
        // warp per slot measured faster (107 against 110-113 us).
        if (mx || K < 8)
            launch(dispatch_scatter_kernel, static_cast<unsigned>((slots + 7) / 8), 256, 0, s, idx, T, K, nt,
                   c.n_experts, bitmap, prefix, offsets, feat, L, mx ? 0 : L, rows_dst, L, perm, inv);
        else
            launch(dispatch_scatter_rows_kernel, static_cast<unsigned>((T + SCATTER_WARPS - 1) / SCATTER_WARPS),
                   32 * SCATTER_WARPS, static_cast<size_t>(SCATTER_WARPS) * L * 2, s, idx, T, K, nt, c.n_experts,
                   bitmap, prefix, offsets, feat, L, L, rows_dst, L, perm, inv);
        if (c.expert_fmt == LMOE_FMT_NVFP4)
            launch(nv_gather_kernel, static_cast<unsigned>((slots + 7) / 8), 256, 0, s, idx, inv, T, K, c.n_experts,
                   feat, L, L, h->at<uint8_t>(p.rows4), h->at<uint8_t>(p.rows_sf4), static_cast<int>(c.max_tokens) * K);
        else if (mx)
            launch(mx_gather_kernel, static_cast<unsigned>((slots + 7) / 8), 256, 0, s, idx, inv, T, K, c.n_experts,
                   feat, L, L, h->at<uint8_t>(p.rows8), L, h->at<uint8_t>(p.rows_sf), mx_ld_sf(L));
    }
    return LMOE_OK;
}

// Expert up (+ activation) and down GEMMs over the sorted rows in the
// workspace, by the tile lists and counts in its header; the outputs replace
// the rows.  need_tc: some expert has more than `small` rows (the grouped GEMMs
// run).
int run_experts(lmoe_handle* h, int small, bool need_tc, cudaStream_t s) {
    const lmoe_config& c = h->c;
    const Plan& p = h->p;
    const int L = c.latent, m = c.m;
    const bool mx = c.expert_fmt != LMOE_FMT_BF16;
    int* hdr = h->at<int>(p.hdr);
    __nv_bfloat16* rows = h->at<__nv_bfloat16>(p.rows);
    __nv_bfloat16* hbuf = h->at<__nv_bfloat16>(p.hbuf);
    int4* mt_list = h->at<int4>(p.mt_list);
    int4* small_list = h->at<int4>(p.small_list);
    GemmArgs base{};
    base.err = hdr + HDR_ERR;
    base.timeout_ns = h->timeout_ns;

    const bool pair = need_tc && h->group_pair && h->group_pair_ok;
    GroupArgs ga{};
    ga.list = h->at<int4>(p.pt_list);
    ga.count = hdr + HDR_PT;
    ga.err = hdr + HDR_ERR;
    ga.timeout_ns = h->timeout_ns;
    // ---------------------------------------------------------------- expert up (+ activation)
    if (pair) {
        // CTA pairs, weight rows as the 256-row operand: each expert's rows in N <= 256 token tiles
        PhaseScope ps(h, PH_UP_TC, s, 1);
        GroupArgs a = ga;
        a.K = L;
        a.n_mt = c.act == LMOE_ACT_SWIGLU ? m / 128 : m / 256;
        a.w_rows_per_expert = h->g * m;
        a.up_offset = m;
        a.out = hbuf;
        a.ld_out = m;
        if (c.act == LMOE_ACT_SWIGLU)
            launch_group<EPI_SWIGLU>(h->w1g16, h->rows32, h->rows64, h->a_rows, h->og_h, a, h->num_sms, s);
        else if (c.act == LMOE_ACT_RELU2)
            launch_group<EPI_RELU2>(h->w1s, h->rows32, h->rows64, h->a_rows, h->og_h, a, h->num_sms, s);
        else launch_group<EPI_BF16>(h->w1s, h->rows32, h->rows64, h->a_rows, h->og_h, a, h->num_sms, s);
    } else if (need_tc) {
        PhaseScope ps(h, PH_UP_TC, s, 1);
        GemmArgs a = base;
        a.K = L;
        a.mt_list = mt_list;
        a.mt_count = hdr + HDR_MT;
        a.b_rows_per_expert = h->g * m;
        a.up_offset = m;
        a.N0 = m;
        a.out0 = hbuf;
        a.ld0 = m;
        if (c.act == LMOE_ACT_SWIGLU) {
            a.n_tiles = (m + 127) / 128;
            launch_gemm<256, EPI_SWIGLU>(h->a_rows, h->w1, h->w1, a, h->num_sms, s, &h->o_h);
        } else if (c.act == LMOE_ACT_RELU2) {
            a.n_tiles = (m + 255) / 256;
            launch_gemm<256, EPI_RELU2>(h->a_rows, h->w1, h->w1, a, h->num_sms, s, &h->o_h);
        } else {
            a.n_tiles = (m + 255) / 256;
            launch_gemm<256, EPI_BF16>(h->a_rows, h->w1, h->w1, a, h->num_sms, s, &h->o_h);
        }
    }
    if (c.expert_fmt == LMOE_FMT_NVFP4) {
        PhaseScope ps(h, PH_UP_STREAM, s, 1);
        NvArgs a{};
        a.K = L;
        a.n_wtiles = m / 128;
        a.list = small_list;
        a.count = hdr + HDR_NSMALL;
        a.w_rows_per_expert = h->g * m;
        a.up_offset = m;
        a.w_sf = static_cast<const uint8_t*>(h->w.w1_scales);
        a.w_g = h->w.w1_gscale;
        a.n_out = m;
        a.out4 = h->at<uint8_t>(p.h4);
        a.out_sf = h->at<uint8_t>(p.h_sf4);
        a.sf_rows = static_cast<int>(c.max_tokens) * c.top_k;
        a.err = hdr + HDR_ERR;
        a.timeout_ns = h->timeout_ns;
        const int epi = c.act == LMOE_ACT_SWIGLU ? EPI_SWIGLU : (c.act == LMOE_ACT_RELU2 ? EPI_RELU2 : EPI_BF16);
        launch_nv_phase(true, epi, h->w1n, h->rows4, h->rows_sf4, a, h->num_sms, s);
    } else if (mx) {
        PhaseScope ps(h, PH_UP_STREAM, s, 1);
        MxArgs a{};
        a.K = L;
        a.n_wtiles = m / 128;
        a.list = small_list;
        a.count = hdr + HDR_NSMALL;
        a.w_rows_per_expert = h->g * m;
        a.up_offset = m;
        a.w_sf = static_cast<const uint8_t*>(h->w.w1_scales);
        a.n_out = m;
        a.out8 = h->at<uint8_t>(p.h8);
        a.out_sf = h->at<uint8_t>(p.h_sf);
        a.ld_out8 = m;
        a.ld_out_sf = mx_ld_sf(m);
        a.err = hdr + HDR_ERR;
        a.timeout_ns = h->timeout_ns;
        const int epi = c.act == LMOE_ACT_SWIGLU ? EPI_SWIGLU : (c.act == LMOE_ACT_RELU2 ? EPI_RELU2 : EPI_BF16);
        launch_mx_phase(true, epi, c.expert_fmt == LMOE_FMT_MXFP4, h->w1q, h->rows8, h->rows_sf, a, h->num_sms, s);
    } else if (small > 0) {
        PhaseScope ps(h, PH_UP_STREAM, s, 1);
        SwapArgs a{};
        a.K = L;
        a.k_splits = 1;
        a.n_wtiles = (m + 127) / 128;
        a.list = small_list;
        a.count = hdr + HDR_NSMALL;
        a.w_rows_per_expert = h->g * m;
        a.up_offset = m;
        a.n_out = m;
        a.out = hbuf;
        a.ld_out = m;
        a.err = hdr + HDR_ERR;
        a.timeout_ns = h->timeout_ns;
        const int epi = c.act == LMOE_ACT_SWIGLU ? EPI_SWIGLU : (c.act == LMOE_ACT_RELU2 ? EPI_RELU2 : EPI_BF16);
        launch_stream(small, epi, h->w1s, h->rows16, h->rows32, a, h->num_sms, s);
    }
    // ---------------------------------------------------------------- expert down (output reuses the gathered rows)
    if (pair) {
        PhaseScope ps(h, PH_DOWN_TC, s, 1);
        GroupArgs a = ga;
        a.K = m;
        a.n_mt = L / 256;
        a.w_rows_per_expert = L;
        a.out = rows;
        a.ld_out = L;
        launch_group<EPI_BF16>(h->w2s, h->h32, h->h64, h->a_h, h->og_rows, a, h->num_sms, s);
    } else if (need_tc) {
        PhaseScope ps(h, PH_DOWN_TC, s, 1);
        GemmArgs a = base;
        a.K = m;
        a.mt_list = mt_list;
        a.mt_count = hdr + HDR_MT;
        a.b_rows_per_expert = L;
        a.N0 = L;
        a.out0 = rows;
        a.ld0 = L;
        a.n_tiles = (L + 255) / 256;
        launch_gemm<256, EPI_BF16>(h->a_h, h->w2, h->w2, a, h->num_sms, s, &h->o_rows);
    }
    if (c.expert_fmt == LMOE_FMT_NVFP4) {
        PhaseScope ps(h, PH_DOWN_STREAM, s, 1);
        NvArgs a{};
        a.K = m;
        a.n_wtiles = L / 128;
        a.list = small_list;
        a.count = hdr + HDR_NSMALL;
        a.w_rows_per_expert = L;
        a.up_offset = 0;
        a.w_sf = static_cast<const uint8_t*>(h->w.w2_scales);
        a.w_g = h->w.w2_gscale;
        a.n_out = L;
        a.out = rows;
        a.ld_out = L;
        a.err = hdr + HDR_ERR;
        a.timeout_ns = h->timeout_ns;
        launch_nv_phase(false, EPI_BF16, h->w2n, h->h4, h->h_sf4, a, h->num_sms, s);
    } else if (mx) {
        PhaseScope ps(h, PH_DOWN_STREAM, s, 1);
        MxArgs a{};
        a.K = m;
        a.n_wtiles = L / 128;
        a.list = small_list;
        a.count = hdr + HDR_NSMALL;
        a.w_rows_per_expert = L;
        a.up_offset = 0;
        a.w_sf = static_cast<const uint8_t*>(h->w.w2_scales);
        a.n_out = L;
        a.out = rows;
        a.ld_out = L;
        a.err = hdr + HDR_ERR;
        a.timeout_ns = h->timeout_ns;
        launch_mx_phase(false, EPI_BF16, c.expert_fmt == LMOE_FMT_MXFP4, h->w2q, h->h8, h->h_sf, a, h->num_sms, s);
    } else if (small > 0) {
        PhaseScope ps(h, PH_DOWN_STREAM, s, 1);
        SwapArgs a{};
        a.K = m;
        a.k_splits = 1;
        a.n_wtiles = (L + 127) / 128;
        a.list = small_list;
        a.count = hdr + HDR_NSMALL;
        a.w_rows_per_expert = L;
        a.up_offset = 0;
        a.n_out = L;
        a.out = rows;
        a.ld_out = L;
        a.err = hdr + HDR_ERR;
        a.timeout_ns = h->timeout_ns;
        launch_stream(small, EPI_BF16, h->w2s, h->h16, h->h32, a, h->num_sms, s);
    }
    return LMOE_OK;
}

// Combine in the latent width of the expert outputs O (the sorted rows of the
// FFN-expert slots, ld = latent), then W_up + residual (joining the shared
// expert's side stream).
int run_back(lmoe_handle* h, const __nv_bfloat16* O, const void* x, void* y, int T, cudaStream_t s) {
    const lmoe_config& c = h->c;
    const Plan& p = h->p;
    const int K = c.top_k, L = c.latent, d = c.d;
    const bool proj = c.has_proj != 0;
    int* hdr = h->at<int>(p.hdr);
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
    __nv_bfloat16* yb = static_cast<__nv_bfloat16*>(y);
    const __nv_bfloat16* feat = proj ? h->at<__nv_bfloat16>(p.z) : xb;
    const __nv_bfloat16* resid = c.shared_m > 0 ? h->at<__nv_bfloat16>(p.s2) : xb;  // x + shared expert, or x
    const int32_t* idx = h->at<int32_t>(p.idx);
    const float* wts = h->at<float>(p.w);
    const int32_t* inv = h->at<int32_t>(p.inv);
    const int m_tiles = (T + 127) / 128;
    GemmArgs base{};
    base.err = hdr + HDR_ERR;
    base.timeout_ns = h->timeout_ns;

    // ---------------------------------------------------------------- combine in the latent width
    {
        PhaseScope ps(h, PH_COMBINE, s, 1);
        __nv_bfloat16* out = proj ? h->at<__nv_bfloat16>(p.yl) : yb;
        if (!proj && c.shared_m > 0 && cudaStreamWaitEvent(s, h->ev_join, 0) != cudaSuccess) return LMOE_ERR_CUDA;
        // small batches: all K' rows in flight per thread (latency); large: 4 (more resident blocks), which
        // measured 72 against 78 us (8 rows) and 83 us (2 rows) on the Nemotron-like prefill
        auto kern = T <= 256 ? combine_kernel<32> : combine_kernel<4>;
        launch(kern, T, 128, 0, s, O, L,
               static_cast<const int32_t*>(inv), static_cast<const int32_t*>(idx), static_cast<const float*>(wts),
               feat, L, static_cast<const __nv_bfloat16*>(h->w.const_vecs), T, K, L, c.n_experts, c.n_zero, c.n_copy,
               proj ? static_cast<const __nv_bfloat16*>(nullptr) : resid, d, out, proj ? L : d);
    }
    // ---------------------------------------------------------------- W_up + residual
    if (proj && c.shared_m > 0 && cudaStreamWaitEvent(s, h->ev_join, 0) != cudaSuccess) return LMOE_ERR_CUDA;
    if (proj && T <= kFewTokenRows) {
        PhaseScope ps(h, PH_WUP, s, 2);
        FewTokenGemm g{&h->wup128, &h->wup128, &h->yl16, &h->yl32, d, 0, L, yb, d, nullptr, 0, resid, d};
        launch_few_token(g, T, h->at<float>(p.partial), kFewTokenMaxSplits, h->num_sms, hdr + HDR_ERR, h->timeout_ns,
                         s);
    } else if (proj) {
        PhaseScope ps(h, PH_WUP, s, 1);
        GemmArgs a = base;
        a.M = T;
        a.K = L;
        a.N0 = d;
        a.out0 = yb;
        a.ld0 = d;
        a.resid = resid;
        a.ld_resid = d;
        if (m_tiles * ((d + 255) / 256) >= h->num_sms) {
            a.n_tiles = (d + 255) / 256;
            CUtensorMap o_y;
            if (!make_map(&o_y, y, T, d, d, 32)) return LMOE_ERR_CUDA;
            launch_gemm_pair<EPI_RESID>(h->a_yl, h->wup128, h->wup128, a, (T + 255) / 256 * a.n_tiles, h->num_sms, s,
                                        &o_y);
        } else {
            a.n_tiles = (d + 63) / 64;
            launch_gemm<64, EPI_RESID>(h->a_yl, h->wup64, h->wup64, a, std::min(h->num_sms, m_tiles * a.n_tiles), s);
        }
    }
    if (cudaGetLastError() != cudaSuccess) return LMOE_ERR_CUDA;
    if (h->prof && h->prof_n < h->prof_max) ++h->prof_n;
    return LMOE_OK;
}

// Experts with at most `small` rows stream their weights.  rows_bound bounds
// the rows of any one expert (the token count of a forward); when every expert
// must stream (rows_bound <= small) the grouped GEMMs are not launched at all.
int choose_small(const lmoe_handle* h, long rows_bound) {
    int small = h->small_max;
    if (small > 0 && rows_bound <= SMALL_MAX) small = rows_bound <= 16 ? 16 : SMALL_MAX;
    if (h->c.expert_fmt != LMOE_FMT_BF16) small = SMALL_MAX;  // block-scaled experts always stream
    return small;
}

// The `small_max` the dispatch builds its lists with: block-scaled experts stream whatever their rows, in
// list entries of at most 32 rows (chunk mode, a negative value); others split by `small`.
int list_small(const lmoe_handle* h, int small) { return h->c.expert_fmt != LMOE_FMT_BF16 ? -SMALL_MAX : small; }

int run_forward(lmoe_handle* h, const void* x, void* y, int T, cudaStream_t s, const lmoe_debug* dbg) {
    const lmoe_config& c = h->c;
    const Plan& p = h->p;
    const int K = c.top_k, L = c.latent, nt = h->n_tot;
    const bool proj = c.has_proj != 0;
    const int small = choose_small(h, T);
    h->last_small = small;
    h->stats_ep = false;
    __nv_bfloat16* rows = h->at<__nv_bfloat16>(p.rows);
    int st = run_front(h, x, T, s, rows, list_small(h, small));
    if (st != LMOE_OK) return st;
    st = run_experts(h, small, c.expert_fmt == LMOE_FMT_BF16 && T > small, s);
    if (st != LMOE_OK) return st;
    st = run_back(h, rows, x, y, T, s);
    if (st != LMOE_OK) return st;

    if (dbg != nullptr) {
        bool ok = true;
        auto cp = [&](void* dst, const void* src, size_t bytes) {
            if (dst) ok &= cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
        };
        cp(dbg->topk_idx, h->at<int32_t>(p.idx), static_cast<size_t>(T) * K * 4);
        cp(dbg->topk_w, h->at<float>(p.w), static_cast<size_t>(T) * K * 4);
        cp(dbg->counts, h->at<int>(p.counts), static_cast<size_t>(nt) * 4);
        cp(dbg->offsets, h->at<int>(p.offsets), static_cast<size_t>(nt + 1) * 4);
        cp(dbg->perm, h->at<int32_t>(p.perm), static_cast<size_t>(T) * K * 4);
        if (proj) {
            cp(dbg->z, h->at<__nv_bfloat16>(p.z), static_cast<size_t>(T) * L * 2);
            cp(dbg->yl, h->at<__nv_bfloat16>(p.yl), static_cast<size_t>(T) * L * 2);
        }
        if (dbg->logits)
            ok &= cudaMemcpy2DAsync(dbg->logits, static_cast<size_t>(nt) * 4, h->at<float>(p.logits), static_cast<size_t>(p.ld_logits) * 4,
                                    static_cast<size_t>(nt) * 4, T, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
        if (!ok) return LMOE_ERR_CUDA;
    }
    return LMOE_OK;
}

constexpr size_t kGraphCache = 8;

// The launch sequence of a captured graph: each node's kind and, for kernels, the function.
bool graph_signature(cudaGraph_t g, std::vector<const void*>& sig) {
    size_t n = 0;
    if (cudaGraphGetNodes(g, nullptr, &n) != cudaSuccess) return false;
    std::vector<cudaGraphNode_t> nodes(n);
    if (n > 0 && cudaGraphGetNodes(g, nodes.data(), &n) != cudaSuccess) return false;
    sig.clear();
    for (size_t i = 0; i < n; ++i) {
        cudaGraphNodeType t;
        if (cudaGraphNodeGetType(nodes[i], &t) != cudaSuccess) return false;
        sig.push_back(reinterpret_cast<const void*>(static_cast<uintptr_t>(t) + 1));
        if (t == cudaGraphNodeTypeKernel) {
            cudaKernelNodeParams kp{};
            if (cudaGraphKernelNodeGetParams(nodes[i], &kp) != cudaSuccess) return false;
            sig.push_back(kp.func);
        }
    }
    return true;
}

// One forward as a CUDA graph.  The launches of run_forward are captured on the handle's own stream and
// replayed on `s` from the executable graph kept for the same launch sequence, updated in place (pointers,
// grid sizes), or from a new one.  A graph launch costs the GPU less per kernel than the same launches issued
// one by one, and the capture costs host time only.
int forward_graph(lmoe_handle* h, const void* x, void* y, int T, cudaStream_t s) {
    if (cudaStreamBeginCapture(h->cap, cudaStreamCaptureModeThreadLocal) != cudaSuccess) return LMOE_ERR_CUDA;
    const int st = run_forward(h, x, y, T, h->cap, nullptr);
    cudaGraph_t g = nullptr;
    const cudaError_t ce = cudaStreamEndCapture(h->cap, &g);
    if (st != LMOE_OK || ce != cudaSuccess || g == nullptr) {
        if (g != nullptr) cudaGraphDestroy(g);
        cudaGetLastError();  // the capture's own error state; the handle stays usable
        return st != LMOE_OK ? st : LMOE_ERR_CUDA;
    }
    std::vector<const void*> sig;
    const bool have_sig = graph_signature(g, sig);
    cudaGetLastError();
    int idx = -1;
    for (size_t i = 0; have_sig && i < h->graphs.size(); ++i)
        if (h->graphs[i].sig == sig) idx = static_cast<int>(i);
    if (idx >= 0) {
        cudaGraphExecUpdateResultInfo info;
        if (cudaGraphExecUpdate(h->graphs[idx].exec, g, &info) != cudaSuccess) {
            cudaGetLastError();  // an update refused for a changed shape is not an error of the forward
            cudaGraphExecDestroy(h->graphs[idx].exec);
            h->graphs.erase(h->graphs.begin() + idx);
            idx = -1;
        }
    }
    if (idx < 0) {
        cudaGraphExec_t e = nullptr;
        if (cudaGraphInstantiate(&e, g, 0) != cudaSuccess) {
            cudaGraphDestroy(g);
            return LMOE_ERR_CUDA;
        }
        if (h->graphs.size() >= kGraphCache) {
            size_t lru = 0;
            for (size_t i = 1; i < h->graphs.size(); ++i)
                if (h->graphs[i].used < h->graphs[lru].used) lru = i;
            cudaGraphExecDestroy(h->graphs[lru].exec);  // freed when a launch still in flight completes
            h->graphs.erase(h->graphs.begin() + lru);
        }
        lmoe_handle::GraphExec ge;
        ge.sig = have_sig ? sig : std::vector<const void*>{};
        ge.exec = e;
        h->graphs.push_back(ge);
        idx = static_cast<int>(h->graphs.size()) - 1;
    }
    cudaGraphDestroy(g);
    h->graphs[idx].used = ++h->graph_tick;
    return cudaGraphLaunch(h->graphs[idx].exec, s) == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

// The graph form is taken for layers whose forward runs on one stream.  A layer with a shared expert forks it
// to a second stream, and its graph measured slower than its direct launches (313 against 304 us on the
// Nemotron-like decode step).  It is also skipped while the caller captures `s` into a graph of its own (the
// launches then go into that capture directly), with phase timing on (its events time single launches) and
// for debug copies.
bool graph_forward_ok(const lmoe_handle* h, cudaStream_t s, const lmoe_debug* dbg) {
    if (!h->use_graph || h->c.shared_m > 0 || h->prof || dbg != nullptr) return false;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return cs == cudaStreamCaptureStatusNone;
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

size_t lmoe_workspace_bytes(const lmoe_config* cfg) {
    if (cfg == nullptr || !config_ok(*cfg)) return 0;
    return make_plan(*cfg).total;
}

int lmoe_create(const lmoe_config* cfg, const lmoe_weights* w, void* workspace, size_t workspace_bytes,
                lmoe_handle** out) {
    if (out == nullptr || cfg == nullptr || w == nullptr) return LMOE_ERR_INVALID_ARG;
    *out = nullptr;
    if (!config_ok(*cfg)) return LMOE_ERR_UNSUPPORTED_SHAPE;
    const lmoe_config& c = *cfg;
    const Plan p = make_plan(c);
    if (workspace == nullptr || workspace_bytes < p.total) return LMOE_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return LMOE_ERR_INVALID_ARG;
    if (w->w_router == nullptr || w->w1 == nullptr || w->w2 == nullptr) return LMOE_ERR_INVALID_ARG;
    if (c.has_proj && (w->w_down == nullptr || w->w_up == nullptr)) return LMOE_ERR_INVALID_ARG;
    if (c.n_const > 0 && w->const_vecs == nullptr) return LMOE_ERR_INVALID_ARG;
    if (c.shared_m > 0 && (w->w_shared1 == nullptr || w->w_shared2 == nullptr)) return LMOE_ERR_INVALID_ARG;
    const void* ptrs[] = {w->w_router, w->router_bias, w->w_down, w->w_up, w->w1, w->w2, w->const_vecs,
                          w->w_shared1, w->w_shared2, w->w1_scales, w->w2_scales, w->w1_gscale, w->w2_gscale};
    for (const void* q : ptrs)
        if (!aligned16(q)) return LMOE_ERR_INVALID_ARG;
    if (c.expert_fmt == LMOE_FMT_NVFP4 && (w->w1_gscale == nullptr || w->w2_gscale == nullptr))
        return LMOE_ERR_INVALID_ARG;
    if (c.expert_fmt != LMOE_FMT_BF16) {
        if (w->w1_scales == nullptr || w->w2_scales == nullptr) return LMOE_ERR_INVALID_ARG;
        // the packed E2M1 copy reads from 32-byte aligned rows
        if (c.expert_fmt == LMOE_FMT_MXFP4 &&
            ((reinterpret_cast<uintptr_t>(w->w1) | reinterpret_cast<uintptr_t>(w->w2)) & 31) != 0)
            return LMOE_ERR_INVALID_ARG;
    }

    lmoe_handle* h = new (std::nothrow) lmoe_handle();
    if (h == nullptr) return LMOE_ERR_INVALID_ARG;
    h->c = c;
    h->w = *w;
    h->ws = static_cast<uint8_t*>(workspace);
    h->p = p;
    h->n_tot = n_total(c);
    h->n_local = n_local_experts(c);
    h->g = c.act == LMOE_ACT_SWIGLU ? 2 : 1;
    if (cudaGetDevice(&h->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess ||
        !set_all_smem_attrs()) {
        delete h;
        return LMOE_ERR_CUDA;
    }
    const int L = c.latent, d = c.d, m = c.m, nt = h->n_tot;
    const int fdim = c.latent_router ? L : d;
    const uint64_t R = static_cast<uint64_t>(c.max_tokens) * c.top_k;
    const uint64_t RC = p.rows_cap;
    bool ok = true;
    ok &= make_map(&h->wr128, w->w_router, nt, fdim, fdim, 128);
    ok &= make_map(&h->wr64, w->w_router, nt, fdim, fdim, 64);
    ok &= make_map(&h->wr256, w->w_router, nt, fdim, fdim, 256);
    if (c.has_proj) {
        ok &= make_map(&h->wdown64, w->w_down, L, d, d, 64);
        ok &= make_map(&h->wdown256, w->w_down, L, d, d, 256);
        ok &= make_map(&h->wup64, w->w_up, d, L, L, 64);
        ok &= make_map(&h->wup256, w->w_up, d, L, L, 256);
        ok &= make_map(&h->a_yl, h->at<void>(p.yl), c.max_tokens, L, L, 128);
        ok &= make_map(&h->a_z, h->at<void>(p.z), c.max_tokens, L, L, 128);
        ok &= make_map(&h->wdown128, w->w_down, L, d, d, 128);
        ok &= make_map(&h->wup128, w->w_up, d, L, L, 128);
        ok &= make_map(&h->z16, h->at<void>(p.z), c.max_tokens, L, L, 16);
        ok &= make_map(&h->z32, h->at<void>(p.z), c.max_tokens, L, L, 32);
        ok &= make_map(&h->yl16, h->at<void>(p.yl), c.max_tokens, L, L, 16);
        ok &= make_map(&h->yl32, h->at<void>(p.yl), c.max_tokens, L, L, 32);
        if (c.latent_router) {
            ok &= make_map(&h->a_zlo, h->at<void>(p.zlo), c.max_tokens, L, L, 128);
            ok &= make_map(&h->zlo16, h->at<void>(p.zlo), c.max_tokens, L, L, 16);
            ok &= make_map(&h->zlo32, h->at<void>(p.zlo), c.max_tokens, L, L, 32);
        }
    }
    const uint64_t w1_rows = static_cast<uint64_t>(h->n_local) * h->g * m, w2_rows = static_cast<uint64_t>(h->n_local) * L;
    if (c.expert_fmt == LMOE_FMT_BF16) {
        ok &= make_map(&h->w1, w->w1, w1_rows, L, L, h->g == 2 ? 128 : 256);
        ok &= make_map(&h->w2, w->w2, w2_rows, m, m, 256);
        ok &= make_map(&h->w1s, w->w1, w1_rows, L, L, 128);
        ok &= make_map(&h->w2s, w->w2, w2_rows, m, m, 128);
    } else if (c.expert_fmt == LMOE_FMT_NVFP4) {
        const uint64_t RT = static_cast<uint64_t>(c.max_tokens) * c.top_k;
        ok &= make_map_u8(&h->w1n, w->w1, w1_rows, L / 2, L / 2, 128, 128, true);
        ok &= make_map_u8(&h->w2n, w->w2, w2_rows, m / 2, m / 2, 128, 128, true);
        ok &= make_map_u8(&h->rows4, h->at<void>(p.rows4), RT, L / 2, L / 2, 128, 32, true);
        ok &= make_map_u8(&h->h4, h->at<void>(p.h4), RT, m / 2, m / 2, 128, 32, true);
        ok &= make_map_nv_sf(&h->rows_sf4, h->at<void>(p.rows_sf4), RT, L / 64);
        ok &= make_map_nv_sf(&h->h_sf4, h->at<void>(p.h_sf4), RT, m / 64);
    } else {
        if (c.expert_fmt == LMOE_FMT_MXFP4) {
            ok &= make_map_e2m1(&h->w1q, w->w1, w1_rows, L);
            ok &= make_map_e2m1(&h->w2q, w->w2, w2_rows, m);
        } else {
            ok &= make_map_u8(&h->w1q, w->w1, w1_rows, L, L, 128, 128, true);
            ok &= make_map_u8(&h->w2q, w->w2, w2_rows, m, m, 128, 128, true);
        }
        ok &= make_map_u8(&h->rows8, h->at<void>(p.rows8), R, L, L, 128, 32, true);
        ok &= make_map_u8(&h->rows_sf, h->at<void>(p.rows_sf), R, mx_ld_sf(L), mx_ld_sf(L), 16, 32, false);
        ok &= make_map_u8(&h->h8, h->at<void>(p.h8), R, m, m, 128, 32, true);
        ok &= make_map_u8(&h->h_sf, h->at<void>(p.h_sf), R, mx_ld_sf(m), mx_ld_sf(m), 16, 32, false);
    }
    ok &= make_map(&h->a_rows, h->at<void>(p.rows), RC, L, L, 128);
    ok &= make_map(&h->a_h, h->at<void>(p.hbuf), RC, m, m, 128);
    ok &= make_map(&h->o_h, h->at<void>(p.hbuf), RC, m, m, 32);
    ok &= make_map(&h->o_rows, h->at<void>(p.rows), RC, L, L, 32);
    h->group_pair_ok = c.expert_fmt == LMOE_FMT_BF16 && L % 256 == 0 && m % (h->g == 2 ? 128 : 256) == 0;
    if (h->group_pair_ok) {
        if (h->g == 2) ok &= make_map_gated(&h->w1g16, w->w1, h->n_local, m, L);
        ok &= make_map_plain(&h->og_h, h->at<void>(p.hbuf), RC, m, m, h->g == 2 ? 16 : 32, 32);
        ok &= make_map_plain(&h->og_rows, h->at<void>(p.rows), RC, L, L, 32, 32);
        ok &= make_map(&h->rows64, h->at<void>(p.rows), RC, L, L, 64);
        ok &= make_map(&h->h64, h->at<void>(p.hbuf), RC, m, m, 64);
    }
    if (c.has_proj) ok &= make_map(&h->o_z, h->at<void>(p.z), c.max_tokens, L, L, 32);
    ok &= make_map(&h->rows16, h->at<void>(p.rows), RC, L, L, 16);
    ok &= make_map(&h->rows32, h->at<void>(p.rows), RC, L, L, 32);
    ok &= make_map(&h->h16, h->at<void>(p.hbuf), RC, m, m, 16);
    ok &= make_map(&h->h32, h->at<void>(p.hbuf), RC, m, m, 32);
    if (c.shared_m > 0) {
        const int ms = c.shared_m, srows = h->g * ms;
        ok &= make_map(&h->ws1_64, w->w_shared1, srows, d, d, h->g == 2 ? 32 : 64);
        ok &= make_map(&h->ws1_256, w->w_shared1, srows, d, d, h->g == 2 ? 128 : 256);
        ok &= make_map(&h->ws1_128, w->w_shared1, srows, d, d, 128);
        ok &= make_map(&h->ws2_64, w->w_shared2, d, ms, ms, 64);
        ok &= make_map(&h->ws2_256, w->w_shared2, d, ms, ms, 256);
        ok &= make_map(&h->ws2_128, w->w_shared2, d, ms, ms, 128);
        ok &= make_map(&h->a_hs, h->at<void>(p.hs), c.max_tokens, ms, ms, 128);
        ok &= make_map(&h->hs16, h->at<void>(p.hs), c.max_tokens, ms, ms, 16);
        ok &= make_map(&h->hs32, h->at<void>(p.hs), c.max_tokens, ms, ms, 32);
        ok &= cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking) == cudaSuccess;
        ok &= cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming) == cudaSuccess;
        ok &= cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming) == cudaSuccess;
    }
    ok &= cudaStreamCreateWithFlags(&h->cap, cudaStreamNonBlocking) == cudaSuccess;
    ok &= cudaMemset(h->at<void>(p.hdr), 0, HDR_WORDS * 4) == cudaSuccess;
    if (!ok) {
        lmoe_destroy(h);
        return LMOE_ERR_CUDA;
    }
    *out = h;
    return LMOE_OK;
}

int lmoe_forward(lmoe_handle* h, const void* x, void* y, int32_t T, void* stream, const lmoe_debug* dbg) {
    if (h == nullptr || h->c.ep_size > 1) return LMOE_ERR_INVALID_ARG;
    if (T < 0 || T > h->c.max_tokens) return LMOE_ERR_TOO_MANY_TOKENS;
    if (T == 0) return LMOE_OK;
    if (x == nullptr || y == nullptr) return LMOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y)) return LMOE_ERR_INVALID_ARG;
    const size_t bytes = static_cast<size_t>(T) * h->c.d * 2;
    const uintptr_t xa = reinterpret_cast<uintptr_t>(x), ya = reinterpret_cast<uintptr_t>(y);
    if (xa < ya + bytes && ya < xa + bytes) return LMOE_ERR_INVALID_ARG;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (graph_forward_ok(h, s, dbg)) return forward_graph(h, x, y, T, s);
    return run_forward(h, x, y, T, s, dbg);
}

// The copy stream and events of the host-buffer forward, made on its first use.
bool host_copy_ready(lmoe_handle* h) {
    if (h->hcopy != nullptr) return true;
    cudaStream_t cs = nullptr;
    cudaEvent_t ev[4] = {nullptr, nullptr, nullptr, nullptr};
    bool ok = cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) == cudaSuccess;
    for (int i = 0; i < 4 && ok; ++i) ok = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {  // nothing half made stays behind
        for (cudaEvent_t e : ev)
            if (e != nullptr) cudaEventDestroy(e);
        if (cs != nullptr) cudaStreamDestroy(cs);
        return false;
    }
    h->ev_in[0] = ev[0], h->ev_in[1] = ev[1], h->ev_used[0] = ev[2], h->ev_used[1] = ev[3];
    h->hcopy = cs;
    return true;
}

int lmoe_forward_host(lmoe_handle* h, const void* x_host, void* y_host, int32_t T, void* stream) {
    if (h == nullptr || h->c.ep_size > 1) return LMOE_ERR_INVALID_ARG;
    if (T < 0 || T > h->c.max_tokens) return LMOE_ERR_TOO_MANY_TOKENS;
    if (T == 0) return LMOE_OK;
    if (x_host == nullptr || y_host == nullptr) return LMOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t bytes = static_cast<size_t>(T) * h->c.d * 2;
    void* yout = h->at<void>(h->p.yout);
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) return LMOE_ERR_CUDA;
    void* xin = h->at<void>(h->p.xin);
    if (cap != cudaStreamCaptureStatusNone || !host_copy_ready(h)) {
        // captured by the caller (or no copy stream): everything in order on `stream`
        if (cudaMemcpyAsync(xin, x_host, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess) return LMOE_ERR_CUDA;
    } else {
        // The input copy goes on the handle's copy stream, into the buffer the forward before last read (its
        // forward has finished with it once ev_used fires); `stream` waits for the copy.  A caller that issues
        // calls back to back thus has each call's copy overlap the previous call's forward.
        const int b = static_cast<int>(h->host_calls & 1);
        xin = h->at<void>(b ? h->p.xin2 : h->p.xin);
        if (cudaStreamWaitEvent(h->hcopy, h->ev_used[b], 0) != cudaSuccess ||
            cudaMemcpyAsync(xin, x_host, bytes, cudaMemcpyHostToDevice, h->hcopy) != cudaSuccess ||
            cudaEventRecord(h->ev_in[b], h->hcopy) != cudaSuccess || cudaStreamWaitEvent(s, h->ev_in[b], 0) != cudaSuccess)
            return LMOE_ERR_CUDA;
        const int rc = graph_forward_ok(h, s, nullptr) ? forward_graph(h, xin, yout, T, s)
                                                       : run_forward(h, xin, yout, T, s, nullptr);
        if (rc != LMOE_OK) return rc;
        if (cudaEventRecord(h->ev_used[b], s) != cudaSuccess) return LMOE_ERR_CUDA;
        ++h->host_calls;
        if (cudaMemcpyAsync(y_host, yout, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess) return LMOE_ERR_CUDA;
        return LMOE_OK;
    }
    const int rc = graph_forward_ok(h, s, nullptr) ? forward_graph(h, xin, yout, T, s) : run_forward(h, xin, yout, T, s, nullptr);
    if (rc != LMOE_OK) return rc;
    if (cudaMemcpyAsync(y_host, yout, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess) return LMOE_ERR_CUDA;
    return LMOE_OK;
}

int lmoe_ep_dispatch(lmoe_handle* h, const void* x, int32_t T, void* send_rows, int32_t* send_counts, void* stream) {
    if (h == nullptr) return LMOE_ERR_INVALID_ARG;
    if (h->c.expert_fmt != LMOE_FMT_BF16) return LMOE_ERR_UNSUPPORTED_SHAPE;
    if (T < 0 || T > h->c.max_tokens) return LMOE_ERR_TOO_MANY_TOKENS;
    if (send_counts == nullptr || !aligned16(send_counts)) return LMOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (cudaMemsetAsync(send_counts, 0, static_cast<size_t>(h->c.n_experts) * 4, s) != cudaSuccess)
            return LMOE_ERR_CUDA;
        h->ep_x = nullptr;
        h->ep_T = 0;
        h->ep_block_rows = 0;
        return LMOE_OK;
    }
    if (x == nullptr || send_rows == nullptr || !aligned16(x) || !aligned16(send_rows)) return LMOE_ERR_INVALID_ARG;
    // the tile lists the sort builds are not used here: the experts stage rebuilds them for the rows it receives
    const int st = run_front(h, x, T, s, static_cast<__nv_bfloat16*>(send_rows), h->small_max);
    if (st != LMOE_OK) return st;
    if (cudaMemcpyAsync(send_counts, h->at<int>(h->p.counts), static_cast<size_t>(h->c.n_experts) * 4,
                        cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return LMOE_ERR_CUDA;
    h->ep_x = x;
    h->ep_T = T;
    h->ep_block_rows = 0;
    return LMOE_OK;
}

int lmoe_ep_experts(lmoe_handle* h, const void* recv_rows, const int32_t* recv_counts, int32_t n_recv,
                    int32_t rows_bound, void* out_rows, void* stream) {
    if (h == nullptr) return LMOE_ERR_INVALID_ARG;
    const lmoe_config& c = h->c;
    if (c.expert_fmt != LMOE_FMT_BF16) return LMOE_ERR_UNSUPPORTED_SHAPE;
    if (n_recv < 0 || static_cast<size_t>(n_recv) > h->p.ep_cap) return LMOE_ERR_TOO_MANY_TOKENS;
    if (n_recv == 0) {  // nothing to compute; the routing statistics show an empty stage
        cudaStream_t s0 = static_cast<cudaStream_t>(stream);
        if (cudaMemsetAsync(h->at<int>(h->p.ep_counts), 0, static_cast<size_t>(h->n_local) * 4, s0) != cudaSuccess ||
            cudaMemsetAsync(h->at<int>(h->p.hdr) + HDR_ROWS, 0, 3 * 4, s0) != cudaSuccess)
            return LMOE_ERR_CUDA;
        h->stats_ep = true;
        return LMOE_OK;
    }
    if (rows_bound < 1) return LMOE_ERR_INVALID_ARG;
    if (recv_rows == nullptr || recv_counts == nullptr || out_rows == nullptr || !aligned16(recv_rows) ||
        !aligned16(recv_counts) || !aligned16(out_rows))
        return LMOE_ERR_INVALID_ARG;
    const Plan& p = h->p;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int ep = ep_ranks(c), nl = h->n_local, L = c.latent;
    const int small = choose_small(h, rows_bound);
    h->last_small = small;
    h->stats_ep = true;
    int* hdr = h->at<int>(p.hdr);
    int* src_off = h->at<int>(p.ep_src);
    int* dst_base = h->at<int>(p.ep_dst);
    int32_t* map = h->at<int32_t>(p.ep_map);
    __nv_bfloat16* rows = h->at<__nv_bfloat16>(p.rows);
    const int n_seg = ep * nl;
    const unsigned grid = static_cast<unsigned>(
        std::min<long>((n_recv + EP_ROWS_PER_PASS - 1) / EP_ROWS_PER_PASS, 8L * h->num_sms));
    {
        PhaseScope ps(h, PH_EP_REGROUP, s, 2);
        launch(ep_prep_kernel, 1, 1024, 0, s, recv_counts, ep, nl, static_cast<int>(n_recv),
               static_cast<int>(rows_bound), small, h->at<int>(p.ep_counts), h->at<int>(p.ep_offsets),
               h->at<int4>(p.mt_list), h->at<int4>(p.small_list), h->at<int4>(p.pt_list), src_off, dst_base, hdr, 0);
        launch(ep_regroup_kernel, grid, 32 * EP_ROWS_PER_PASS, static_cast<size_t>(2 * n_seg + 1) * 4, s,
               static_cast<const __nv_bfloat16*>(recv_rows), static_cast<int>(n_recv), L,
               static_cast<const int*>(src_off), static_cast<const int*>(dst_base), n_seg,
               static_cast<const int*>(hdr), rows, map);
    }
    const int st = run_experts(h, small, rows_bound > small, s);
    if (st != LMOE_OK) return st;
    {
        PhaseScope ps(h, PH_EP_REGROUP, s, 1);
        launch(ep_unregroup_kernel, grid, 32 * EP_ROWS_PER_PASS, 0, s, static_cast<const __nv_bfloat16*>(rows),
               static_cast<const int32_t*>(map), static_cast<int>(n_recv), L, static_cast<const int*>(hdr),
               static_cast<__nv_bfloat16*>(out_rows));
    }
    return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

// ---------------------------------------------------------------- the block exchange
namespace {
// The most rows one rank can send to one other rank in a forward of up to max_tokens tokens: each token has
// at most min(top_k, n_local) slots on a rank's experts (a token's experts are distinct).
int64_t ep_block_cap(const lmoe_handle* h) {
    return static_cast<int64_t>(h->c.max_tokens) * std::min(h->c.top_k, h->n_local);
}
}  // namespace

int64_t lmoe_ep_block_rows(lmoe_handle* h) {
    return h == nullptr ? 0 : ep_block_cap(h);
}

int lmoe_ep_dispatch_blocks(lmoe_handle* h, const void* x, int32_t T, void* send_blocks, int32_t block_rows,
                            int32_t* send_counts, void* stream) {
    if (h == nullptr) return LMOE_ERR_INVALID_ARG;
    if (h->c.expert_fmt != LMOE_FMT_BF16) return LMOE_ERR_UNSUPPORTED_SHAPE;
    if (T < 0 || T > h->c.max_tokens) return LMOE_ERR_TOO_MANY_TOKENS;
    if (block_rows < 1 || block_rows < static_cast<int64_t>(T) * std::min(h->c.top_k, h->n_local) ||
        block_rows > ep_block_cap(h))
        return LMOE_ERR_INVALID_ARG;
    if (send_counts == nullptr || !aligned16(send_counts)) return LMOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (cudaMemsetAsync(send_counts, 0, static_cast<size_t>(h->c.n_experts) * 4, s) != cudaSuccess)
            return LMOE_ERR_CUDA;
        h->ep_x = nullptr;
        h->ep_T = 0;
        h->ep_block_rows = block_rows;
        return LMOE_OK;
    }
    if (x == nullptr || send_blocks == nullptr || !aligned16(x) || !aligned16(send_blocks)) return LMOE_ERR_INVALID_ARG;
    const Plan& p = h->p;
    __nv_bfloat16* packed = h->at<__nv_bfloat16>(p.rows);
    const int st = run_front(h, x, T, s, packed, h->small_max);
    if (st != LMOE_OK) return st;
    const int ep = ep_ranks(h->c), nl = h->n_local, L = h->c.latent;
    const int n_rows = T * h->c.top_k;
    {
        PhaseScope ps(h, PH_EP_REGROUP, s, 1);
        launch(ep_block_copy_kernel, static_cast<unsigned>(std::min<long>((n_rows + EP_ROWS_PER_PASS - 1) / EP_ROWS_PER_PASS,
                                                                          8L * h->num_sms)),
               32 * EP_ROWS_PER_PASS, 0, s, static_cast<const __nv_bfloat16*>(packed),
               static_cast<__nv_bfloat16*>(send_blocks), static_cast<const int*>(h->at<int>(p.offsets)), nl, ep,
               static_cast<int>(block_rows), n_rows, L, 1);
    }
    if (cudaMemcpyAsync(send_counts, h->at<int>(p.counts), static_cast<size_t>(h->c.n_experts) * 4,
                        cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return LMOE_ERR_CUDA;
    h->ep_x = x;
    h->ep_T = T;
    h->ep_block_rows = block_rows;
    return LMOE_OK;
}

int lmoe_ep_experts_blocks(lmoe_handle* h, const void* recv_blocks, int32_t block_rows, const int32_t* recv_counts,
                           int32_t rows_bound, void* out_blocks, void* stream) {
    if (h == nullptr) return LMOE_ERR_INVALID_ARG;
    const lmoe_config& c = h->c;
    if (c.expert_fmt != LMOE_FMT_BF16) return LMOE_ERR_UNSUPPORTED_SHAPE;
    if (block_rows < 1 || block_rows > ep_block_cap(h) || rows_bound < 1) return LMOE_ERR_INVALID_ARG;
    if (recv_blocks == nullptr || recv_counts == nullptr || out_blocks == nullptr || !aligned16(recv_blocks) ||
        !aligned16(recv_counts) || !aligned16(out_blocks))
        return LMOE_ERR_INVALID_ARG;
    const Plan& p = h->p;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int ep = ep_ranks(c), nl = h->n_local, L = c.latent;
    const int n = ep * block_rows;  // the received buffer's rows, used or not
    const int small = choose_small(h, rows_bound);
    h->last_small = small;
    h->stats_ep = true;
    int* hdr = h->at<int>(p.hdr);
    int* src_off = h->at<int>(p.ep_src);
    int* dst_base = h->at<int>(p.ep_dst);
    int32_t* map = h->at<int32_t>(p.ep_map);
    __nv_bfloat16* rows = h->at<__nv_bfloat16>(p.rows);
    const unsigned grid =
        static_cast<unsigned>(std::min<long>((n + EP_ROWS_PER_PASS - 1) / EP_ROWS_PER_PASS, 8L * h->num_sms));
    {
        PhaseScope ps(h, PH_EP_REGROUP, s, 2);
        launch(ep_prep_kernel, 1, 1024, 0, s, recv_counts, ep, nl, n, static_cast<int>(rows_bound), small,
               h->at<int>(p.ep_counts), h->at<int>(p.ep_offsets), h->at<int4>(p.mt_list), h->at<int4>(p.small_list),
               h->at<int4>(p.pt_list), src_off, dst_base, hdr, static_cast<int>(block_rows));
        launch(ep_regroup_blocks_kernel, grid, 32 * EP_ROWS_PER_PASS, 0, s,
               static_cast<const __nv_bfloat16*>(recv_blocks), static_cast<int>(block_rows), L, recv_counts,
               static_cast<const int*>(src_off), static_cast<const int*>(dst_base), ep, nl,
               static_cast<const int*>(hdr), rows, map);
    }
    const int st = run_experts(h, small, rows_bound > small, s);
    if (st != LMOE_OK) return st;
    {
        PhaseScope ps(h, PH_EP_REGROUP, s, 1);
        launch(ep_unregroup_blocks_kernel, grid, 32 * EP_ROWS_PER_PASS, 0, s, static_cast<const __nv_bfloat16*>(rows),
               static_cast<const int32_t*>(map), n, L, static_cast<const int*>(hdr),
               static_cast<__nv_bfloat16*>(out_blocks));
    }
    return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

int lmoe_ep_combine_blocks(lmoe_handle* h, const void* ret_blocks, void* y, void* stream) {
    if (h == nullptr || h->ep_T < 0 || h->ep_block_rows < 1) return LMOE_ERR_INVALID_ARG;
    if (h->c.expert_fmt != LMOE_FMT_BF16) return LMOE_ERR_UNSUPPORTED_SHAPE;
    const int T = h->ep_T;
    const void* x = h->ep_x;
    if (T == 0) {
        h->ep_T = -1;
        h->ep_block_rows = 0;
        return LMOE_OK;
    }
    if (ret_blocks == nullptr || y == nullptr || !aligned16(ret_blocks) || !aligned16(y)) return LMOE_ERR_INVALID_ARG;
    const size_t bytes = static_cast<size_t>(T) * h->c.d * 2;
    const uintptr_t xa = reinterpret_cast<uintptr_t>(x), ya = reinterpret_cast<uintptr_t>(y);
    if (xa < ya + bytes && ya < xa + bytes) return LMOE_ERR_INVALID_ARG;
    const Plan& p = h->p;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int n_rows = T * h->c.top_k;
    __nv_bfloat16* packed = h->at<__nv_bfloat16>(p.rows);
    {
        PhaseScope ps(h, PH_EP_REGROUP, s, 1);
        launch(ep_block_copy_kernel, static_cast<unsigned>(std::min<long>((n_rows + EP_ROWS_PER_PASS - 1) / EP_ROWS_PER_PASS,
                                                                          8L * h->num_sms)),
               32 * EP_ROWS_PER_PASS, 0, s, static_cast<const __nv_bfloat16*>(ret_blocks), packed,
               static_cast<const int*>(h->at<int>(p.offsets)), h->n_local, ep_ranks(h->c),
               static_cast<int>(h->ep_block_rows), n_rows, h->c.latent, 0);
    }
    h->ep_T = -1;
    h->ep_block_rows = 0;
    return run_back(h, packed, x, y, T, s);
}

int lmoe_ep_combine(lmoe_handle* h, const void* ret_rows, void* y, void* stream) {
    if (h == nullptr || h->ep_T < 0 || h->ep_block_rows != 0) return LMOE_ERR_INVALID_ARG;
    if (h->c.expert_fmt != LMOE_FMT_BF16) return LMOE_ERR_UNSUPPORTED_SHAPE;
    const int T = h->ep_T;
    const void* x = h->ep_x;
    if (T == 0) {
        h->ep_T = -1;
        return LMOE_OK;
    }
    if (ret_rows == nullptr || y == nullptr || !aligned16(ret_rows) || !aligned16(y)) return LMOE_ERR_INVALID_ARG;
    const size_t bytes = static_cast<size_t>(T) * h->c.d * 2;
    const uintptr_t xa = reinterpret_cast<uintptr_t>(x), ya = reinterpret_cast<uintptr_t>(y);
    if (xa < ya + bytes && ya < xa + bytes) return LMOE_ERR_INVALID_ARG;
    h->ep_T = -1;
    return run_back(h, static_cast<const __nv_bfloat16*>(ret_rows), x, y, T, static_cast<cudaStream_t>(stream));
}

int lmoe_last_error(lmoe_handle* h) {
    if (h == nullptr) return LMOE_ERR_INVALID_ARG;
    int err = 0;
    int* dev = h->at<int>(h->p.hdr) + HDR_ERR;
    if (cudaMemcpy(&err, dev, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return LMOE_ERR_CUDA;
    if (err != 0 && cudaMemset(dev, 0, 4) != cudaSuccess) return LMOE_ERR_CUDA;
    if (err & DEVERR_TIMEOUT) return LMOE_ERR_TIMEOUT;
    if (err & (DEVERR_BAD_INDEX | DEVERR_REPEATED_INDEX)) return LMOE_ERR_BAD_INDEX;
    if (err & DEVERR_BAD_COUNTS) return LMOE_ERR_BAD_COUNTS;
    return LMOE_OK;
}

void lmoe_destroy(lmoe_handle* h) {
    if (h == nullptr) return;
    free_events(h);
    if (h->ev_fork) cudaEventDestroy(h->ev_fork);
    if (h->ev_join) cudaEventDestroy(h->ev_join);
    if (h->side) cudaStreamDestroy(h->side);
    for (int b = 0; b < 2; ++b) {
        if (h->ev_in[b]) cudaEventDestroy(h->ev_in[b]);
        if (h->ev_used[b]) cudaEventDestroy(h->ev_used[b]);
    }
    if (h->hcopy) cudaStreamDestroy(h->hcopy);
    for (auto& ge : h->graphs)
        if (ge.exec) cudaGraphExecDestroy(ge.exec);  // one still in flight is freed when it completes
    if (h->cap) cudaStreamDestroy(h->cap);
    delete h;
}

const char* lmoe_status_string(int status) {
    switch (status) {
        case LMOE_OK: return "ok";
        case LMOE_ERR_INVALID_ARG: return "invalid argument";
        case LMOE_ERR_UNSUPPORTED_SHAPE: return "unsupported layer shape";
        case LMOE_ERR_TOO_MANY_TOKENS: return "token count outside [0, max_tokens]";
        case LMOE_ERR_CUDA: return "CUDA call failed";
        case LMOE_ERR_TIMEOUT: return "a bounded wait inside a kernel gave up";
        case LMOE_ERR_BAD_INDEX: return "expert id out of range";
        case LMOE_ERR_WORKSPACE: return "workspace missing or too small";
        case LMOE_ERR_BAD_COUNTS: return "received row counts inconsistent";
        default: return "unknown status";
    }
}

int lmoe_set_profiling(lmoe_handle* h, int enable, int max_forwards) {
    if (h == nullptr || (enable && max_forwards < 1)) return LMOE_ERR_INVALID_ARG;
    free_events(h);
    h->prof = enable != 0;
    if (!h->prof) return LMOE_OK;
    const size_t n = static_cast<size_t>(max_forwards) * PH_COUNT;
    h->ev.assign(2 * n, nullptr);
    h->launches.assign(n, 0);
    for (auto& e : h->ev)
        if (cudaEventCreate(&e) != cudaSuccess) {
            free_events(h);
            h->prof = false;
            return LMOE_ERR_CUDA;
        }
    h->prof_max = max_forwards;
    h->prof_n = 0;
    return LMOE_OK;
}

int lmoe_phase_times(lmoe_handle* h, float* ms, int32_t* launches) {
    if (h == nullptr) return LMOE_ERR_INVALID_ARG;
    std::vector<float> acc(PH_COUNT, 0.f);
    std::vector<int32_t> nl(PH_COUNT, 0);
    for (int f = 0; f < h->prof_n; ++f)
        for (int ph = 0; ph < PH_COUNT; ++ph) {
            const size_t i = static_cast<size_t>(f) * PH_COUNT + ph;
            if (h->launches[i] == 0) continue;
            float t = 0.f;
            if (cudaEventElapsedTime(&t, h->ev[2 * i], h->ev[2 * i + 1]) != cudaSuccess) return LMOE_ERR_CUDA;
            acc[ph] += t;
            nl[ph] += h->launches[i];
            h->launches[i] = 0;
        }
    h->prof_n = 0;
    for (int ph = 0; ph < PH_COUNT; ++ph) {
        if (ms) ms[ph] = acc[ph];
        if (launches) launches[ph] = nl[ph];
    }
    return LMOE_OK;
}

int lmoe_num_phases(void) { return PH_COUNT; }

const char* lmoe_phase_name(int phase) { return (phase >= 0 && phase < PH_COUNT) ? kPhaseNames[phase] : nullptr; }

int lmoe_routing_stats(lmoe_handle* h, int32_t* out8) {
    if (h == nullptr || out8 == nullptr) return LMOE_ERR_INVALID_ARG;
    int hdr[HDR_WORDS];
    // after an expert-parallel experts stage: the local experts' received rows; else the forward's routing
    const int n_ffn = h->stats_ep ? h->n_local : h->c.n_experts;
    std::vector<int> counts(n_ffn);
    if (cudaMemcpy(hdr, h->at<int>(h->p.hdr), sizeof hdr, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(counts.data(), h->at<int>(h->stats_ep ? h->p.ep_counts : h->p.counts), counts.size() * 4,
                   cudaMemcpyDeviceToHost) != cudaSuccess)
        return LMOE_ERR_CUDA;
    int touched = 0, st_experts = 0, st_rows = 0, tc_experts = 0, tc_rows = 0;
    const bool all_stream = h->c.expert_fmt != LMOE_FMT_BF16;
    for (int e = 0; e < n_ffn; ++e) {
        const int n = counts[e];
        touched += n > 0;
        if (n > 0 && (all_stream || n <= h->last_small)) {
            ++st_experts;
            st_rows += n;
        } else if (n > h->last_small) {
            ++tc_experts;
            tc_rows += n;
        }
    }
    out8[0] = hdr[HDR_ROWS];
    out8[1] = touched;
    out8[2] = hdr[HDR_MT];
    out8[3] = hdr[HDR_NSMALL];
    out8[4] = st_rows;
    out8[5] = tc_experts;
    out8[6] = tc_rows;
    out8[7] = h->last_small;
    return LMOE_OK;
}

int lmoe_set_small_rows(lmoe_handle* h, int32_t rows) {
    if (h == nullptr || rows < 0 || rows > SMALL_MAX) return LMOE_ERR_INVALID_ARG;
    h->small_max = rows;
    return LMOE_OK;
}

int lmoe_set_graph_launch(lmoe_handle* h, int enable) {
    if (h == nullptr || (enable != 0 && enable != 1)) return LMOE_ERR_INVALID_ARG;
    h->use_graph = enable;
    return LMOE_OK;
}

int lmoe_set_grouped_gemm(lmoe_handle* h, int kind) {
    if (h == nullptr || (kind != 0 && kind != 1)) return LMOE_ERR_INVALID_ARG;
    h->group_pair = kind;
    return LMOE_OK;
}

int lmoe_set_wait_timeout(lmoe_handle* h, uint64_t ns) {
    if (h == nullptr || ns == 0) return LMOE_ERR_INVALID_ARG;
    h->timeout_ns = ns;
    return LMOE_OK;
}

int lmoe_selftest_wait(lmoe_handle* h, uint64_t timeout_ns, void* stream) {
    if (h == nullptr || timeout_ns == 0 || timeout_ns > 2000000000ull) return LMOE_ERR_INVALID_ARG;
    wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(h->at<int>(h->p.hdr) + HDR_ERR, timeout_ns);
    return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

int lmoe_gemm_bf16(const void* A, const void* B, void* C, int32_t M, int32_t N, int32_t K, void* stream, int* err_word) {
    if (A == nullptr || B == nullptr || C == nullptr || err_word == nullptr) return LMOE_ERR_INVALID_ARG;
    if (M < 0 || N < 64 || N % 64 != 0 || K < 64 || K % 64 != 0 || K > 65536) return LMOE_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(A) || !aligned16(B) || !aligned16(C)) return LMOE_ERR_INVALID_ARG;
    if (M == 0) return LMOE_OK;
    static std::once_flag attr_once;
    static bool attr_ok = false;
    std::call_once(attr_once, [] { attr_ok = set_all_smem_attrs(); });
    if (!attr_ok) return LMOE_ERR_CUDA;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return LMOE_ERR_CUDA;
    const int m_tiles = (M + 127) / 128;
    const bool big = static_cast<long long>(m_tiles) * ((N + 255) / 256) >= sms;
    CUtensorMap ma, mb;
    // large problems run on CTA pairs (256 x 256 tiles; each CTA loads 128 of the B rows)
    CUtensorMap mc;
    if (!make_map(&ma, A, M, K, K, 128) || !make_map(&mb, B, N, K, K, big ? 128 : 64) || !make_map(&mc, C, M, N, N, 32))
        return LMOE_ERR_CUDA;
    GemmArgs a{};
    a.M = M;
    a.K = K;
    a.N0 = N;
    a.out0 = static_cast<__nv_bfloat16*>(C);
    a.ld0 = N;
    a.err = err_word;
    a.timeout_ns = 1000000000ull;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (big) {
        a.n_tiles = (N + 255) / 256;
        launch_gemm_pair<EPI_BF16>(ma, mb, mb, a, static_cast<int>(std::min<long long>(sms, (M + 255LL) / 256 * a.n_tiles)),
                                   sms, s, &mc);
    } else {
        a.n_tiles = (N + 63) / 64;
        launch_gemm<64, EPI_BF16>(ma, mb, mb, a, std::min<long long>(sms, static_cast<long long>(m_tiles) * a.n_tiles), s);
    }
    return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

int lmoe_nvfp4_encode_weights(const void* w, int32_t n_mats, int64_t rows_per_mat, int32_t K, void* codes,
                              void* scales, float* gscale, void* stream) {
    if (n_mats < 1 || n_mats > 65535 || rows_per_mat < 128 || rows_per_mat % 128 != 0 || K < 64 || K % 64 != 0 ||
        static_cast<long long>(n_mats) * rows_per_mat * K > (1LL << 40))
        return LMOE_ERR_UNSUPPORTED_SHAPE;
    if (w == nullptr || codes == nullptr || scales == nullptr || gscale == nullptr || !aligned16(w) ||
        !aligned16(codes) || !aligned16(scales) || !aligned16(gscale))
        return LMOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t* gbits = reinterpret_cast<uint32_t*>(gscale);
    if (cudaMemsetAsync(gbits, 0, static_cast<size_t>(n_mats) * 4, s) != cudaSuccess) return LMOE_ERR_CUDA;
    const long long per_mat = rows_per_mat * K;
    const unsigned gx = static_cast<unsigned>(std::min<long long>((per_mat / 8 + 255) / 256, 256));
    nv_amax_kernel<<<dim3(gx, static_cast<unsigned>(n_mats)), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(w),
                                                                          per_mat, gbits);
    nv_tensor_scale_kernel<<<(n_mats + 255) / 256, 256, 0, s>>>(gbits, n_mats);
    const long long rows = static_cast<long long>(n_mats) * rows_per_mat;
    const long long blocks = rows * (K / 16);
    nv_encode_weights_kernel<<<static_cast<unsigned>((blocks + 255) / 256), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(w), rows, rows_per_mat, K, gscale, static_cast<uint8_t*>(codes),
        static_cast<uint8_t*>(scales));
    return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

int lmoe_mx_encode_weights(const void* w, int64_t rows, int32_t K, int32_t fmt, void* codes, void* scales,
                           void* stream) {
    if (fmt != LMOE_FMT_MXFP8 && fmt != LMOE_FMT_MXFP4) return LMOE_ERR_UNSUPPORTED_SHAPE;
    if (rows < 0 || rows % 128 != 0 || K < 128 || K % 128 != 0 || K > 65536) return LMOE_ERR_UNSUPPORTED_SHAPE;
    if (rows == 0) return LMOE_OK;
    if (w == nullptr || codes == nullptr || scales == nullptr) return LMOE_ERR_INVALID_ARG;
    if (!aligned16(w) || !aligned16(codes) || !aligned16(scales)) return LMOE_ERR_INVALID_ARG;
    const long long blocks = rows * (K / 32);
    const unsigned grid = static_cast<unsigned>((blocks + 255) / 256);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const __nv_bfloat16* wb = static_cast<const __nv_bfloat16*>(w);
    // a plain launch: this kernel does not wait on a predecessor (no programmatic dependent launch)
    if (fmt == LMOE_FMT_MXFP4)
        mx_encode_weights_kernel<true><<<grid, 256, 0, s>>>(wb, rows, K, static_cast<uint8_t*>(codes),
                                                            static_cast<uint8_t*>(scales));
    else
        mx_encode_weights_kernel<false><<<grid, 256, 0, s>>>(wb, rows, K, static_cast<uint8_t*>(codes),
                                                             static_cast<uint8_t*>(scales));
    return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

}  // extern "C"
