// C ABI of the sbsa library (declared in include/sbsa.h): argument checking, tensor-map
// encoding, workspace carving and kernel launches.  All compute is in the kernels of
// pool.cuh, select.cuh, attn.cuh, rope.cuh, fp8.cuh, nvfp4.cuh and ulysses.cuh; nothing here
// touches tensor data on the host.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/sbsa.h"
#include "attn.cuh"
#include "common.cuh"
#include "fp8.cuh"
#include "nvfp4.cuh"
#include "pool.cuh"
#include "ptx.cuh"
#include "rope.cuh"
#include "select.cuh"
#include "ulysses.cuh"

// 1 (default): the NVFP4 GEMM on CTA pairs (256 x 256 tiles, 38 KB loaded per SM per K-tile);
// 0: one CTA per 128 x 256 tile (54 KB).  Both parity-tested; on 32,768 x 15,360 x 5,120 the
// pair kernel takes 1.15 ms, the one-CTA kernel 1.33 ms (the L2 -> SM load path bounds both).
#ifndef SBSA_NVFP4_PAIR
#define SBSA_NVFP4_PAIR 1
#endif

namespace sbsa {
namespace {

thread_local char t_errmsg[512] = "";

sbsa_status fail(sbsa_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_errmsg, sizeof t_errmsg, fmt, ap);
    va_end(ap);
    return st;
}

sbsa_status ok() {
    t_errmsg[0] = '\0';
    return SBSA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kMaxBlocks = 2048;

sbsa_status check_shape(const sbsa_shape* s) {
    if (!s) return fail(SBSA_ERR_INVALID_ARG, "shape is NULL");
    if (s->batch < 1 || s->heads < 1 || s->seq_len < 1)
        return fail(SBSA_ERR_INVALID_ARG, "batch, heads and seq_len must be >= 1");
    if (s->head_dim != 64 && s->head_dim != 128)
        return fail(SBSA_ERR_UNSUPPORTED, "head_dim %d not in {64, 128}", s->head_dim);
    if (s->block_size != 64 && s->block_size != 128)
        return fail(SBSA_ERR_UNSUPPORTED, "block_size %d not in {64, 128}", s->block_size);
    const long long want = (static_cast<long long>(s->seq_len) + s->block_size - 1) / s->block_size * s->block_size;
    if (s->seq_len_padded != want)
        return fail(SBSA_ERR_INVALID_ARG, "seq_len_padded %d must be seq_len %d rounded up to block_size %d (= %lld)",
                    s->seq_len_padded, s->seq_len, s->block_size, want);
    const long long nb = s->seq_len_padded / s->block_size;
    if (nb > kMaxBlocks) return fail(SBSA_ERR_UNSUPPORTED, "%lld blocks exceed the limit %d", nb, kMaxBlocks);
    const long long rows = static_cast<long long>(s->batch) * s->heads * s->seq_len_padded;
    if (rows >= (1ll << 31)) return fail(SBSA_ERR_UNSUPPORTED, "batch*heads*seq_len_padded must be < 2^31");
    return SBSA_OK;
}

int num_blocks(const sbsa_shape* s) { return s->seq_len_padded / s->block_size; }
long long num_rows(const sbsa_shape* s) { return static_cast<long long>(s->batch) * s->heads * num_blocks(s); }

sbsa_status check_k(const sbsa_shape* s, int32_t k) {
    const int nb = num_blocks(s);
    if (k < 1 || k > nb) return fail(SBSA_ERR_INVALID_ARG, "k_keep %d not in [1, %d]", k, nb);
    if (num_rows(s) * k >= (1ll << 31)) return fail(SBSA_ERR_UNSUPPORTED, "B*H*nb*k_keep must be < 2^31");
    return SBSA_OK;
}

sbsa_status cuda_fail(cudaError_t e, const char* what) {
    return fail(SBSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ---------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2D view [rows][d] of a bf16 tensor, box {64, box_rows}, 128-byte swizzle.
sbsa_status make_map(CUtensorMap* m, const void* base, long long rows, int d, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(SBSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t es[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SBSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return SBSA_OK;
}

// e4m3 codes [rows][128] viewed as a 2D tensor, box = 128 channels (128 B) x box_rows
sbsa_status make_map_codes(CUtensorMap* m, const void* base, long long rows, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(SBSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {128};
    cuuint32_t box[2] = {128, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t es[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SBSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return SBSA_OK;
}

// fp32 block means [rows][128] viewed as a 2D tensor, box = 32 channels (128 B) x box_rows
sbsa_status make_map_means(CUtensorMap* m, const float* base, long long rows, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(SBSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {128 * 4};
    cuuint32_t box[2] = {32, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t es[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SBSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return SBSA_OK;
}

// NVFP4 codes [rows][K/2] bytes, box = 128 bytes (256 codes) x box_rows, 128-byte swizzle;
// rows beyond the matrix read as zero codes.
sbsa_status make_map_fp4(CUtensorMap* m, const void* base, long long rows, int K, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(SBSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
    cuuint32_t box[2] = {128, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t es[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SBSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return SBSA_OK;
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 148;
    return n > 0 ? n : 148;
}

std::atomic<unsigned int> g_epoch{1};

// Light-Ulysses dimensions of one head chunk, or an error
sbsa_status ulysses_dims(const sbsa_ulysses_shape* s, int32_t head0, int32_t head_chunk, UlyssesDims* u) {
    if (!s) return fail(SBSA_ERR_INVALID_ARG, "shape is NULL");
    if (s->world < 1 || s->tokens < 1 || s->heads < 1) return fail(SBSA_ERR_INVALID_ARG, "world, tokens, heads >= 1");
    if (s->head_dim != kUlyD) return fail(SBSA_ERR_UNSUPPORTED, "head_dim must be 128");
    if (s->tokens % s->world || s->heads % s->world)
        return fail(SBSA_ERR_INVALID_ARG, "tokens and heads must be multiples of world");
    if (s->tokens_padded < s->tokens) return fail(SBSA_ERR_INVALID_ARG, "tokens_padded < tokens");
    const int hg = s->heads / s->world;
    if (head0 < 0 || head_chunk < 1 || head0 + head_chunk > hg)
        return fail(SBSA_ERR_INVALID_ARG, "head chunk outside [0, heads / world)");
    u->G = s->world;
    u->Lr = s->tokens / s->world;
    u->L = s->tokens;
    u->Lp = s->tokens_padded;
    u->H = s->heads;
    u->Hg = hg;
    u->h0 = head0;
    u->hc = head_chunk;
    // the kernels index rows in 32 bits
    const long long rows = static_cast<long long>(u->G) * u->Lr * 3 * u->hc + 3LL * u->hc * (u->Lp - u->L);
    if (rows >= (1LL << 31)) return fail(SBSA_ERR_UNSUPPORTED, "head chunk of 2^31 rows or more");
    const uint32_t pad = static_cast<uint32_t>(u->Lp - u->L);
    u->by_qkv_peer = make_fastdiv(static_cast<uint32_t>(u->Lr) * 3u * static_cast<uint32_t>(u->hc));
    u->by_o_peer = make_fastdiv(static_cast<uint32_t>(u->Lr) * static_cast<uint32_t>(u->hc));
    u->by_hc = make_fastdiv(static_cast<uint32_t>(u->hc));
    u->by_pad = make_fastdiv(pad > 0 ? pad : 1u);  // used only when there are padded tokens
    u->by_pad_hc = make_fastdiv(pad > 0 ? pad * static_cast<uint32_t>(u->hc) : 1u);
    return SBSA_OK;
}


// ---------------------------------------------------------------- launchers
sbsa_status launch_pool(const sbsa_shape* s, const void* q, const void* k, float* qm, float* km, cudaStream_t st) {
    const long long units = num_rows(s);
    const dim3 grid(static_cast<unsigned>(2 * units));
    const int L = s->seq_len, Lp = s->seq_len_padded, nb = num_blocks(s);
    const uint4* q4 = static_cast<const uint4*>(q);
    const uint4* k4 = static_cast<const uint4*>(k);
    if (s->head_dim == 128) {
        if (s->block_size == 128) pool_kernel<128, 128><<<grid, 256, 0, st>>>(q4, k4, qm, km, L, Lp, nb, units);
        else pool_kernel<128, 64><<<grid, 256, 0, st>>>(q4, k4, qm, km, L, Lp, nb, units);
    } else {
        if (s->block_size == 128) pool_kernel<64, 128><<<grid, 256, 0, st>>>(q4, k4, qm, km, L, Lp, nb, units);
        else pool_kernel<64, 64><<<grid, 256, 0, st>>>(q4, k4, qm, km, L, Lp, nb, units);
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SBSA_OK : cuda_fail(e, "pool launch");
}

sbsa_status launch_rope_pool(const sbsa_shape* s, int gt, int gh, int gw, const float2* table, const void* q,
                             const void* k, void* qo, void* ko, float* qm, float* km, cudaStream_t st) {
    const long long units = num_rows(s);
    const dim3 grid(static_cast<unsigned>(2 * units));
    const int L = s->seq_len, Lp = s->seq_len_padded, nb = num_blocks(s);
    const unsigned int epoch = g_epoch.fetch_add(1);
    auto q4 = static_cast<const uint4*>(q);
    auto k4 = static_cast<const uint4*>(k);
    auto qo4 = static_cast<uint4*>(qo);
    auto ko4 = static_cast<uint4*>(ko);
    if (s->head_dim == 128) {
        if (s->block_size == 128)
            rope_pool_kernel<128, 128><<<grid, 256, 0, st>>>(q4, k4, qo4, ko4, table, qm, km, L, Lp, nb, gh, gw, gt, units, epoch);
        else
            rope_pool_kernel<128, 64><<<grid, 256, 0, st>>>(q4, k4, qo4, ko4, table, qm, km, L, Lp, nb, gh, gw, gt, units, epoch);
    } else {
        if (s->block_size == 128)
            rope_pool_kernel<64, 128><<<grid, 256, 0, st>>>(q4, k4, qo4, ko4, table, qm, km, L, Lp, nb, gh, gw, gt, units, epoch);
        else
            rope_pool_kernel<64, 64><<<grid, 256, 0, st>>>(q4, k4, qo4, ko4, table, qm, km, L, Lp, nb, gh, gw, gt, units, epoch);
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SBSA_OK : cuda_fail(e, "rope+pool launch");
}

sbsa_status launch_quantize(const sbsa_shape* s, const void* q, const void* k, const float* smooth, void* q8,
                            void* k8, float* qs, float* ks, cudaStream_t st) {
    const long long units = num_rows(s);
    const dim3 grid(static_cast<unsigned>(2 * units));
    const int L = s->seq_len, Lp = s->seq_len_padded, nb = num_blocks(s);
    const unsigned int epoch = g_epoch.fetch_add(1);
    auto q4 = static_cast<const uint4*>(q);
    auto k4 = static_cast<const uint4*>(k);
    auto q2 = static_cast<uint2*>(q8);
    auto k2 = static_cast<uint2*>(k8);
    if (s->block_size == 128)
        quantize_kernel<128, 128><<<grid, 256, 0, st>>>(q4, k4, smooth, q2, k2, qs, ks, L, Lp, nb, units, epoch);
    else
        quantize_kernel<128, 64><<<grid, 256, 0, st>>>(q4, k4, smooth, q2, k2, qs, ks, L, Lp, nb, units, epoch);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SBSA_OK : cuda_fail(e, "quantize launch");
}

template <int D, int KPL>
sbsa_status launch_select_t(const sbsa_shape* s, const float* qm, const float* km, int k, int32_t* rp, int32_t* ci,
                            cudaStream_t st) {
    constexpr int QT = 16;
    const int nb = num_blocks(s);
    const size_t smem = static_cast<size_t>(QT) * D * 4 + static_cast<size_t>(QT) * 32 * KPL * 4;
    auto kern = select_kernel<D, QT, KPL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_fail(e, "select smem attribute");
    const dim3 grid((nb + QT - 1) / QT, static_cast<unsigned>(s->batch * s->heads));
    kern<<<grid, 256, smem, st>>>(qm, km, nb, k, rp, ci, num_rows(s));
    e = cudaGetLastError();
    return e == cudaSuccess ? SBSA_OK : cuda_fail(e, "select launch");
}

template <int KPL>
sbsa_status launch_select_tc(const sbsa_shape* s, const float* qm, const float* km, int k, int32_t* rp, int32_t* ci,
                             cudaStream_t st) {
    const int nb = num_blocks(s);
    CUtensorMap mq, mk;
    sbsa_status r;
    if ((r = make_map_means(&mq, qm, num_rows(s), kSelTcRows)) != SBSA_OK) return r;
    if ((r = make_map_means(&mk, km, num_rows(s), 128)) != SBSA_OK) return r;
    SelTcParams p;
    p.nb = nb;
    p.k_keep = k;
    p.n_rows = num_rows(s);
    p.epoch = g_epoch.fetch_add(1);
    auto kern = select_tc_kernel<KPL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSelTcSmemBytes));
    if (e != cudaSuccess) return cuda_fail(e, "select smem attribute");
    const dim3 grid((nb + kSelTcRows - 1) / kSelTcRows, static_cast<unsigned>(s->batch * s->heads));
    kern<<<grid, kSelTcThreads, kSelTcSmemBytes, st>>>(mq, mk, rp, ci, p);
    e = cudaGetLastError();
    return e == cudaSuccess ? SBSA_OK : cuda_fail(e, "select launch");
}

template <int D>
sbsa_status launch_select_d(const sbsa_shape* s, const float* qm, const float* km, int k, int32_t* rp, int32_t* ci,
                            cudaStream_t st) {
    const int nb = num_blocks(s);
    if constexpr (D == 128) {
        // tensor-core scores (head_dim 128, up to 1024 blocks)
        if (nb <= 64) return launch_select_tc<2>(s, qm, km, k, rp, ci, st);
        if (nb <= 256) return launch_select_tc<8>(s, qm, km, k, rp, ci, st);
        if (nb <= 512) return launch_select_tc<16>(s, qm, km, k, rp, ci, st);
        if (nb <= 1024) return launch_select_tc<32>(s, qm, km, k, rp, ci, st);
    }
    if (nb <= 64) return launch_select_t<D, 2>(s, qm, km, k, rp, ci, st);
    if (nb <= 256) return launch_select_t<D, 8>(s, qm, km, k, rp, ci, st);
    if (nb <= 512) return launch_select_t<D, 16>(s, qm, km, k, rp, ci, st);
    if (nb <= 1024) return launch_select_t<D, 32>(s, qm, km, k, rp, ci, st);
    return launch_select_t<D, 64>(s, qm, km, k, rp, ci, st);
}

sbsa_status launch_select(const sbsa_shape* s, const float* qm, const float* km, int k, int32_t* rp, int32_t* ci,
                          cudaStream_t st) {
    return s->head_dim == 128 ? launch_select_d<128>(s, qm, km, k, rp, ci, st)
                              : launch_select_d<64>(s, qm, km, k, rp, ci, st);
}

template <int D, int BLK, bool FP8 = false>
sbsa_status launch_attn_t(const sbsa_shape* s, const void* q, const void* k, const void* v, const int32_t* rp,
                          const int32_t* ci, float scale, void* o, cudaStream_t st, const float* q_scale = nullptr,
                          const float* k_scale = nullptr) {
    using C = AttnCfg<D, BLK, FP8>;
    const long long rows = static_cast<long long>(s->batch) * s->heads * s->seq_len_padded;
    CUtensorMap mq, mk, mv;
    sbsa_status r;
    if constexpr (FP8) {
        if ((r = make_map_codes(&mq, q, rows, 128)) != SBSA_OK) return r;
        if ((r = make_map_codes(&mk, k, rows, BLK)) != SBSA_OK) return r;
    } else {
        if ((r = make_map(&mq, q, rows, D, 128)) != SBSA_OK) return r;
        if ((r = make_map(&mk, k, rows, D, BLK)) != SBSA_OK) return r;
    }
    if ((r = make_map(&mv, v, rows, D, BLK)) != SBSA_OK) return r;
    AttnParams p;
    p.row_ptr = rp;
    p.col_idx = ci;
    p.o = static_cast<__nv_bfloat16*>(o);
    // paired query blocks (block 64): one unit per two neighbouring query blocks
    p.units_per_bh = C::kPaired ? (num_blocks(s) + 1) / 2 : num_blocks(s);
    p.units = static_cast<long long>(s->batch) * s->heads * p.units_per_bh;
    p.L = s->seq_len;
    p.Lp = s->seq_len_padded;
    p.nb = num_blocks(s);
    p.scale_log2 = std::fabs(scale) * 1.4426950408889634f;
    p.neg_scale = scale < 0.f ? 1 : 0;
    p.epoch = g_epoch.fetch_add(1);
    p.q_scale = q_scale;
    p.k_scale = k_scale;
    p.prefetch_dist = sm_count();
    auto kern = attn_kernel<D, BLK, FP8>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "attention smem attribute");
    kern<<<static_cast<unsigned>(p.units), C::kThreads, C::kSmemBytes, st>>>(mq, mk, mv, p);
    e = cudaGetLastError();
    return e == cudaSuccess ? SBSA_OK : cuda_fail(e, "attention launch");
}

sbsa_status launch_attn(const sbsa_shape* s, const void* q, const void* k, const void* v, const int32_t* rp,
                        const int32_t* ci, float scale, void* o, cudaStream_t st) {
    if (s->head_dim == 128)
        return s->block_size == 128 ? launch_attn_t<128, 128>(s, q, k, v, rp, ci, scale, o, st)
                                    : launch_attn_t<128, 64>(s, q, k, v, rp, ci, scale, o, st);
    return s->block_size == 128 ? launch_attn_t<64, 128>(s, q, k, v, rp, ci, scale, o, st)
                                : launch_attn_t<64, 64>(s, q, k, v, rp, ci, scale, o, st);
}

float resolve_scale(const sbsa_shape* s, float scale) {
    return scale == 0.f ? 1.0f / std::sqrt(static_cast<float>(s->head_dim)) : scale;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsLayout {
    size_t q_mean, k_mean, row_ptr, col_idx, total;
};

WsLayout ws_layout(const sbsa_shape* s, int k) {
    WsLayout w;
    const size_t means = static_cast<size_t>(num_rows(s)) * s->head_dim * sizeof(float);
    w.q_mean = 0;
    w.k_mean = align256(means);
    w.row_ptr = w.k_mean + align256(means);
    w.col_idx = w.row_ptr + align256((static_cast<size_t>(num_rows(s)) + 1) * sizeof(int32_t));
    w.total = w.col_idx + align256(static_cast<size_t>(num_rows(s)) * k * sizeof(int32_t));
    return w;
}

// ---------------------------------------------------------------- CSR validation
__global__ void validate_csr_kernel(const int32_t* row_ptr, const int32_t* col_idx, long long nrows, long long nnz,
                                    int nb, int require_diag, unsigned int* bad) {
    const long long r = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
    if (r > nrows) return;
    if (r == nrows) {
        if (row_ptr[nrows] != nnz || row_ptr[0] != 0) atomicOr(bad, 1u);
        return;
    }
    const long long a = row_ptr[r], b = row_ptr[r + 1];
    if (a < 0 || b < a || b > nnz) { atomicOr(bad, 1u); return; }
    const int diag = static_cast<int>(r % nb);
    bool has_diag = false;
    int prev = -1;
    for (long long e = a; e < b; ++e) {
        const int j = col_idx[e];
        if (j < 0 || j >= nb || j <= prev) { atomicOr(bad, 1u); return; }
        has_diag |= (j == diag);
        prev = j;
    }
    if (require_diag && !has_diag) atomicOr(bad, 1u);
}

}  // namespace

// ---------------------------------------------------------------- allocation-free forward
// Scratch for sbsa_forward_noalloc: block means and the CSR block list live in this
// fixed module-scope array instead of a caller-provided workspace.  Every GPU that
// loads the library reserves it for the life of the process.  Host code must never
// hand the symbol itself to a kernel (on the host it is only a stand-in); its device
// address is looked up with cudaGetSymbolAddress in the current context on every call
// (a lookup, not an allocation), so the address stays right after a device reset or a
// context switch, which load the module again.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
// Device address of the scratch array in the current context.
sbsa_status noalloc_scratch(void** out) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
    *out = p;
    return SBSA_OK;
}
}  // namespace
}  // namespace sbsa

using namespace sbsa;

extern "C" {

int32_t sbsa_version(void) { return 200; }

const char* sbsa_status_string(sbsa_status st) {
    switch (st) {
        case SBSA_OK: return "SBSA_OK";
        case SBSA_ERR_INVALID_ARG: return "SBSA_ERR_INVALID_ARG";
        case SBSA_ERR_UNSUPPORTED: return "SBSA_ERR_UNSUPPORTED";
        case SBSA_ERR_WORKSPACE: return "SBSA_ERR_WORKSPACE";
        case SBSA_ERR_CUDA: return "SBSA_ERR_CUDA";
        case SBSA_ERR_TIMEOUT: return "SBSA_ERR_TIMEOUT";
        case SBSA_ERR_BAD_INDEX: return "SBSA_ERR_BAD_INDEX";
    }
    return "SBSA_ERR_UNKNOWN";
}

const char* sbsa_last_error_message(void) { return t_errmsg; }

int32_t sbsa_keep_blocks(int32_t num_blocks, double keep_fraction) {
    if (num_blocks < 1 || !std::isfinite(keep_fraction)) return 0;
    double k = std::floor(keep_fraction * num_blocks + 0.5);
    if (k < 1) k = 1;
    if (k > num_blocks) k = num_blocks;
    return static_cast<int32_t>(k);
}

size_t sbsa_workspace_bytes(const sbsa_shape* shape, int32_t k_keep) {
    if (check_shape(shape) != SBSA_OK || check_k(shape, k_keep) != SBSA_OK) return 0;
    return ws_layout(shape, k_keep).total;
}

sbsa_status sbsa_pool_qk(const sbsa_shape* shape, const void* q, const void* k, float* q_mean, float* k_mean,
                         void* stream) {
    sbsa_status r = check_shape(shape);
    if (r != SBSA_OK) return r;
    if (!q || !k || !q_mean || !k_mean) return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(q_mean) || !aligned16(k_mean))
        return fail(SBSA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    if ((r = launch_pool(shape, q, k, q_mean, k_mean, static_cast<cudaStream_t>(stream))) != SBSA_OK) return r;
    return ok();
}

size_t sbsa_rope_table_floats(int32_t head_dim, int32_t grid_t, int32_t grid_h, int32_t grid_w) {
    if ((head_dim != 64 && head_dim != 128) || grid_t < 1 || grid_h < 1 || grid_w < 1) return 0;
    return static_cast<size_t>(2 * rope_table_entries(head_dim, grid_t, grid_h, grid_w));
}

sbsa_status sbsa_rope_table_init(int32_t head_dim, int32_t grid_t, int32_t grid_h, int32_t grid_w, double theta,
                                 float* table, void* stream) {
    if (sbsa_rope_table_floats(head_dim, grid_t, grid_h, grid_w) == 0)
        return fail(SBSA_ERR_INVALID_ARG, "head_dim must be 64 or 128 and the grid sizes >= 1");
    if (!(theta > 1.0) || !std::isfinite(theta)) return fail(SBSA_ERR_INVALID_ARG, "theta must be finite and > 1");
    if (!table || (reinterpret_cast<uintptr_t>(table) & 7u)) return fail(SBSA_ERR_INVALID_ARG, "table must be 8-byte aligned");
    const long long n = rope_table_entries(head_dim, grid_t, grid_h, grid_w);
    rope_table_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        head_dim, grid_t, grid_h, grid_w, theta, reinterpret_cast<float2*>(table), n);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "rope table launch");
    return ok();
}

sbsa_status sbsa_rope_pool_qk(const sbsa_shape* shape, int32_t grid_t, int32_t grid_h, int32_t grid_w,
                              const float* table, const void* q, const void* k, void* q_out, void* k_out,
                              float* q_mean, float* k_mean, void* stream) {
    sbsa_status r = check_shape(shape);
    if (r != SBSA_OK) return r;
    if (grid_t < 1 || grid_h < 1 || grid_w < 1 ||
        static_cast<long long>(grid_t) * grid_h * grid_w != static_cast<long long>(shape->seq_len))
        return fail(SBSA_ERR_INVALID_ARG, "grid_t * grid_h * grid_w must equal seq_len");
    if (!q || !k || !q_out || !k_out || !q_mean || !k_mean || !table) return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(q_out) || !aligned16(k_out) || !aligned16(q_mean) ||
        !aligned16(k_mean))
        return fail(SBSA_ERR_INVALID_ARG, "tensors and means must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(table) & 7u) return fail(SBSA_ERR_INVALID_ARG, "table must be 8-byte aligned");
    if ((r = launch_rope_pool(shape, grid_t, grid_h, grid_w, reinterpret_cast<const float2*>(table), q, k, q_out,
                              k_out, q_mean, k_mean, static_cast<cudaStream_t>(stream))) != SBSA_OK)
        return r;
    return ok();
}

sbsa_status sbsa_key_mean(const sbsa_shape* shape, const float* k_mean, float* out, void* stream) {
    sbsa_status r = check_shape(shape);
    if (r != SBSA_OK) return r;
    if (!k_mean || !out) return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    key_mean_kernel<<<static_cast<unsigned>(static_cast<long long>(shape->batch) * shape->heads), shape->head_dim, 0,
                      static_cast<cudaStream_t>(stream)>>>(k_mean, out, shape->head_dim, num_blocks(shape),
                                                            shape->block_size, shape->seq_len);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "key mean launch");
    return ok();
}

sbsa_status sbsa_quantize_qk_fp8(const sbsa_shape* shape, const void* q, const void* k, const float* k_smooth,
                                 void* q8, void* k8, float* q_scale, float* k_scale, void* stream) {
    sbsa_status r = check_shape(shape);
    if (r != SBSA_OK) return r;
    if (shape->head_dim != 128) return fail(SBSA_ERR_UNSUPPORTED, "the FP8 path needs head_dim 128");
    if (!q || !k || !q8 || !k8 || !q_scale || !k_scale) return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(q8) || !aligned16(k8))
        return fail(SBSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
    if (((reinterpret_cast<uintptr_t>(q_scale) | reinterpret_cast<uintptr_t>(k_scale) |
          reinterpret_cast<uintptr_t>(k_smooth)) & 3u))
        return fail(SBSA_ERR_INVALID_ARG, "scales and smoothing vector must be 4-byte aligned");
    if ((r = launch_quantize(shape, q, k, k_smooth, q8, k8, q_scale, k_scale, static_cast<cudaStream_t>(stream))) !=
        SBSA_OK)
        return r;
    return ok();
}

sbsa_status sbsa_attention_fwd_fp8(const sbsa_shape* shape, const void* q8, const void* k8, const void* v,
                                   const float* q_scale, const float* k_scale, const int32_t* row_ptr,
                                   const int32_t* col_idx, float scale, void* o, void* stream) {
    sbsa_status r = check_shape(shape);
    if (r != SBSA_OK) return r;
    if (shape->head_dim != 128) return fail(SBSA_ERR_UNSUPPORTED, "the FP8 path needs head_dim 128");
    if (!q8 || !k8 || !v || !o || !q_scale || !k_scale || !row_ptr || !col_idx)
        return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(q8) || !aligned16(k8) || !aligned16(v) || !aligned16(o))
        return fail(SBSA_ERR_INVALID_ARG, "q8, k8, v, o must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(row_ptr) | reinterpret_cast<uintptr_t>(col_idx) |
         reinterpret_cast<uintptr_t>(q_scale) | reinterpret_cast<uintptr_t>(k_scale)) & 3u)
        return fail(SBSA_ERR_INVALID_ARG, "row_ptr, col_idx and the scales must be 4-byte aligned");
    if (!std::isfinite(scale)) return fail(SBSA_ERR_INVALID_ARG, "scale must be finite");
    const float sc = resolve_scale(shape, scale);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    r = shape->block_size == 128
            ? launch_attn_t<128, 128, true>(shape, q8, k8, v, row_ptr, col_idx, sc, o, st, q_scale, k_scale)
            : launch_attn_t<128, 64, true>(shape, q8, k8, v, row_ptr, col_idx, sc, o, st, q_scale, k_scale);
    if (r != SBSA_OK) return r;
    return ok();
}

size_t sbsa_ulysses_qkv_bytes(const sbsa_ulysses_shape* shape, int32_t head_chunk) {
    UlyssesDims u;
    if (ulysses_dims(shape, 0, head_chunk, &u) != SBSA_OK) return 0;
    return static_cast<size_t>(u.G) * ulysses_qkv_slice_bytes(u);
}

size_t sbsa_ulysses_o_bytes(const sbsa_ulysses_shape* shape, int32_t head_chunk) {
    UlyssesDims u;
    if (ulysses_dims(shape, 0, head_chunk, &u) != SBSA_OK) return 0;
    return static_cast<size_t>(u.G) * ulysses_o_slice_bytes(u);
}

sbsa_status sbsa_ulysses_pack_qkv(const sbsa_ulysses_shape* shape, int32_t head0, int32_t head_chunk, const void* x,
                                  void* send, void* stream) {
    UlyssesDims u;
    sbsa_status r = ulysses_dims(shape, head0, head_chunk, &u);
    if (r != SBSA_OK) return r;
    if (!x || !send) return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(x) || !aligned16(send)) return fail(SBSA_ERR_INVALID_ARG, "x and send must be 16-byte aligned");
    const long long warps = static_cast<long long>(u.G) * u.Lr * 3 * u.hc;
    const long long grid = (warps + kUlyRowsPerCta - 1) / kUlyRowsPerCta;
    ulysses_pack_qkv_kernel<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<uint8_t*>(send), u);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ok() : cuda_fail(e, "ulysses pack launch");
}

sbsa_status sbsa_ulysses_unpack_qkv(const sbsa_ulysses_shape* shape, int32_t head0, int32_t head_chunk,
                                    const void* recv, void* q, void* k, void* v, void* stream) {
    UlyssesDims u;
    sbsa_status r = ulysses_dims(shape, head0, head_chunk, &u);
    if (r != SBSA_OK) return r;
    if (!recv || !q || !k || !v) return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(recv) || !aligned16(q) || !aligned16(k) || !aligned16(v))
        return fail(SBSA_ERR_INVALID_ARG, "recv, q, k, v must be 16-byte aligned");
    const long long warps = static_cast<long long>(u.G) * u.Lr * 3 * u.hc + 3LL * u.hc * (u.Lp - u.L);
    const long long grid = (warps + kUlyRowsPerCta - 1) / kUlyRowsPerCta;
    ulysses_unpack_qkv_kernel<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint8_t*>(recv), static_cast<__nv_bfloat16*>(q), static_cast<__nv_bfloat16*>(k),
        static_cast<__nv_bfloat16*>(v), u);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ok() : cuda_fail(e, "ulysses unpack launch");
}

sbsa_status sbsa_ulysses_pack_o(const sbsa_ulysses_shape* shape, int32_t head0, int32_t head_chunk, const void* o,
                                void* send, void* stream) {
    UlyssesDims u;
    sbsa_status r = ulysses_dims(shape, head0, head_chunk, &u);
    if (r != SBSA_OK) return r;
    if (!o || !send) return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(o) || !aligned16(send)) return fail(SBSA_ERR_INVALID_ARG, "o and send must be 16-byte aligned");
    const long long warps = static_cast<long long>(u.G) * u.Lr * u.hc;
    const long long grid = (warps + kUlyRowsPerCta - 1) / kUlyRowsPerCta;
    ulysses_pack_o_kernel<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<uint8_t*>(send), u);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ok() : cuda_fail(e, "ulysses pack_o launch");
}

sbsa_status sbsa_ulysses_unpack_o(const sbsa_ulysses_shape* shape, int32_t head0, int32_t head_chunk,
                                  const void* recv, void* y, void* stream) {
    UlyssesDims u;
    sbsa_status r = ulysses_dims(shape, head0, head_chunk, &u);
    if (r != SBSA_OK) return r;
    if (!recv || !y) return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(recv) || !aligned16(y)) return fail(SBSA_ERR_INVALID_ARG, "recv and y must be 16-byte aligned");
    const long long warps = static_cast<long long>(u.G) * u.Lr * u.hc;
    const long long grid = (warps + kUlyRowsPerCta - 1) / kUlyRowsPerCta;
    ulysses_unpack_o_kernel<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint8_t*>(recv), static_cast<__nv_bfloat16*>(y), u);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ok() : cuda_fail(e, "ulysses unpack_o launch");
}

sbsa_status sbsa_ulysses_put_qkv(const sbsa_ulysses_shape* shape, int32_t head0, int32_t head_chunk, const void* x,
                                 const uint64_t* peer_bases, uint64_t recv_offset, int32_t rank, void* stream) {
    UlyssesDims u;
    sbsa_status r = ulysses_dims(shape, head0, head_chunk, &u);
    if (r != SBSA_OK) return r;
    if (!x || !peer_bases) return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(x) || (reinterpret_cast<uintptr_t>(peer_bases) & 7u) || (recv_offset & 15u))
        return fail(SBSA_ERR_INVALID_ARG, "x 16-byte aligned, peer_bases 8-byte aligned, recv_offset a multiple of 16");
    if (rank < 0 || rank >= u.G) return fail(SBSA_ERR_INVALID_ARG, "rank outside [0, world)");
    const PeerDst pd{reinterpret_cast<const unsigned long long*>(peer_bases), recv_offset, rank};
    const long long rows = static_cast<long long>(u.G) * u.Lr * 3 * u.hc;
    const long long tiles = (rows + kUlyRowsPerCta - 1) / kUlyRowsPerCta;
    const long long grid = tiles < 8LL * sm_count() ? tiles : 8LL * sm_count();  // one fence per CTA: few CTAs
    ulysses_put_qkv_kernel<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16*>(x), pd, u);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ok() : cuda_fail(e, "ulysses put_qkv launch");
}

sbsa_status sbsa_ulysses_put_o(const sbsa_ulysses_shape* shape, int32_t head0, int32_t head_chunk, const void* o,
                               const uint64_t* peer_bases, uint64_t recv_offset, int32_t rank, void* stream) {
    UlyssesDims u;
    sbsa_status r = ulysses_dims(shape, head0, head_chunk, &u);
    if (r != SBSA_OK) return r;
    if (!o || !peer_bases) return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(o) || (reinterpret_cast<uintptr_t>(peer_bases) & 7u) || (recv_offset & 15u))
        return fail(SBSA_ERR_INVALID_ARG, "o 16-byte aligned, peer_bases 8-byte aligned, recv_offset a multiple of 16");
    if (rank < 0 || rank >= u.G) return fail(SBSA_ERR_INVALID_ARG, "rank outside [0, world)");
    const PeerDst pd{reinterpret_cast<const unsigned long long*>(peer_bases), recv_offset, rank};
    const long long rows = static_cast<long long>(u.G) * u.Lr * u.hc;
    const long long tiles = (rows + kUlyRowsPerCta - 1) / kUlyRowsPerCta;
    const long long grid = tiles < 8LL * sm_count() ? tiles : 8LL * sm_count();  // one fence per CTA: few CTAs
    ulysses_put_o_kernel<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16*>(o), pd, u);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ok() : cuda_fail(e, "ulysses put_o launch");
}

sbsa_status sbsa_peer_signal(const uint64_t* peer_bases, uint64_t flag_offset, int32_t rank, int32_t world,
                             uint32_t value, void* stream) {
    if (!peer_bases) return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    if (world < 1 || world > 1024 || rank < 0 || rank >= world)
        return fail(SBSA_ERR_INVALID_ARG, "world in [1, 1024] and rank in [0, world) required");
    if ((reinterpret_cast<uintptr_t>(peer_bases) & 7u) || (flag_offset & 3u))
        return fail(SBSA_ERR_INVALID_ARG, "peer_bases 8-byte aligned, flag_offset a multiple of 4");
    peer_signal_kernel<<<1, 1024, 0, static_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const unsigned long long*>(peer_bases), flag_offset, rank, world, value);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ok() : cuda_fail(e, "peer signal launch");
}

sbsa_status sbsa_peer_wait(const uint32_t* flags, int32_t world, uint32_t value, double timeout_s, void* stream) {
    if (!flags) return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    if (world < 1 || world > 1024) return fail(SBSA_ERR_INVALID_ARG, "world in [1, 1024] required");
    if (reinterpret_cast<uintptr_t>(flags) & 3u) return fail(SBSA_ERR_INVALID_ARG, "flags must be 4-byte aligned");
    if (!(timeout_s > 0.0) || timeout_s > 60.0) return fail(SBSA_ERR_INVALID_ARG, "timeout_s in (0, 60] required");
    const unsigned long long limit = static_cast<unsigned long long>(timeout_s * 1e9);
    peer_wait_kernel<<<1, 1024, 0, static_cast<cudaStream_t>(stream)>>>(flags, world, value, limit);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ok() : cuda_fail(e, "peer wait launch");
}

size_t sbsa_nvfp4_scale_bytes(int64_t rows, int32_t cols) {
    if (rows < 1 || cols < 64 || cols % 64) return 0;
    return static_cast<size_t>((rows + 127) / 128 * 128) * static_cast<size_t>(cols / 16);
}

sbsa_status sbsa_nvfp4_amax(const void* x, int64_t rows, int32_t cols, float* amax, void* stream) {
    if (!x || !amax) return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    if (rows < 1 || cols < 8 || cols % 8) return fail(SBSA_ERR_INVALID_ARG, "rows >= 1 and cols a multiple of 8 required");
    if (!aligned16(x) || (reinterpret_cast<uintptr_t>(amax) & 3u))
        return fail(SBSA_ERR_INVALID_ARG, "x must be 16-byte and amax 4-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float), st);
    if (e != cudaSuccess) return cuda_fail(e, "amax reset");
    const long long n8 = rows * static_cast<long long>(cols) / 8;
    const long long want = (n8 + 255) / 256;
    const unsigned grid = static_cast<unsigned>(want < 8LL * sm_count() ? want : 8LL * sm_count());
    nvfp4_amax_kernel<<<grid, 256, 0, st>>>(static_cast<const uint4*>(x), n8, reinterpret_cast<unsigned int*>(amax));
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "amax launch");
    return ok();
}

sbsa_status sbsa_nvfp4_quantize(const void* x, int64_t rows, int32_t cols, const float* amax, void* codes,
                                void* scales, void* stream) {
    if (!x || !amax || !codes || !scales) return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    if (rows < 1 || cols < 64 || cols % 64) return fail(SBSA_ERR_INVALID_ARG, "rows >= 1 and cols a multiple of 64 required");
    if (!aligned16(x) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(amax) & 3u))
        return fail(SBSA_ERR_INVALID_ARG, "x and codes must be 16-byte aligned, amax 4-byte aligned");
    const long long rows_p = (rows + 127) / 128 * 128;
    const long long n_threads = rows_p * (cols / 16);
    const long long grid = (n_threads + 255) / 256;
    if (grid > 0x7FFFFFFFLL) return fail(SBSA_ERR_UNSUPPORTED, "matrix too large");
    nvfp4_quantize_kernel<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(x), amax, static_cast<uint2*>(codes), static_cast<uint8_t*>(scales), rows, cols,
        n_threads);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "nvfp4 quantize launch");
    return ok();
}

sbsa_status sbsa_nvfp4_gemm(int32_t m, int32_t n, int32_t k, const void* a, const void* a_scales, const float* a_amax,
                            const void* b, const void* b_scales, const float* b_amax, const float* bias, void* c,
                            void* stream) {
    if (!a || !a_scales || !a_amax || !b || !b_scales || !b_amax || !c) return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    if (m < 1 || n < 8 || n % 8 || k < kFp4TileK || k % kFp4TileK)
        return fail(SBSA_ERR_INVALID_ARG, "need m >= 1, n a multiple of 8, k a multiple of 256");
    if (!aligned16(a) || !aligned16(b) || !aligned16(c) || !aligned16(a_scales) || !aligned16(b_scales))
        return fail(SBSA_ERR_INVALID_ARG, "codes, scales and c must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(a_amax) | reinterpret_cast<uintptr_t>(b_amax) |
         reinterpret_cast<uintptr_t>(bias)) & 3u)
        return fail(SBSA_ERR_INVALID_ARG, "amax and bias must be 4-byte aligned");
#if SBSA_NVFP4_PAIR
    {
        // pairs of CTAs, 256 x 256 tiles
        CUtensorMap ma, mb;
        sbsa_status r;
        Nvfp4Gemm2Params q;
        q.sfa = static_cast<const uint8_t*>(a_scales);
        q.sfb = static_cast<const uint8_t*>(b_scales);
        q.amax_a = a_amax;
        q.amax_b = b_amax;
        q.bias = bias;
        q.c = static_cast<__nv_bfloat16*>(c);
        q.M = m;
        q.N = n;
        q.K = k;
        q.tiles_m = (m + 255) / 256;
        q.tiles_n = (n + 255) / 256;
        q.groups_a = (m + 127) / 128;
        q.groups_b = (n + 127) / 128;
        q.epoch = g_epoch.fetch_add(1);
        if ((r = make_map_fp4(&ma, a, m, k, 128)) != SBSA_OK) return r;
        if ((r = make_map_fp4(&mb, b, n, k, 128)) != SBSA_OK) return r;
        const long long tiles = static_cast<long long>(q.tiles_m) * q.tiles_n;
        if (tiles > 0x3FFFFFFFLL) return fail(SBSA_ERR_UNSUPPORTED, "too many tiles");
        const int pairs = static_cast<int>(tiles < sm_count() / 2 ? tiles : sm_count() / 2);
        cudaError_t e = cudaFuncSetAttribute(nvfp4_gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kF2SmemBytes);
        if (e != cudaSuccess) return cuda_fail(e, "nvfp4 gemm smem attribute");
        nvfp4_gemm_pair_kernel<<<2 * pairs, kFp4Threads, kF2SmemBytes, static_cast<cudaStream_t>(stream)>>>(ma, mb, q);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "nvfp4 gemm launch");
        return ok();
    }
#endif
    CUtensorMap ma, mb;
    sbsa_status r;
    if ((r = make_map_fp4(&ma, a, m, k, kFp4TileM)) != SBSA_OK) return r;
    if ((r = make_map_fp4(&mb, b, n, k, kFp4TileN)) != SBSA_OK) return r;
    Nvfp4GemmParams p;
    p.sfa = static_cast<const uint8_t*>(a_scales);
    p.sfb = static_cast<const uint8_t*>(b_scales);
    p.amax_a = a_amax;
    p.amax_b = b_amax;
    p.bias = bias;
    p.c = static_cast<__nv_bfloat16*>(c);
    p.M = m;
    p.N = n;
    p.K = k;
    p.tiles_m = (m + kFp4TileM - 1) / kFp4TileM;
    p.tiles_n = (n + kFp4TileN - 1) / kFp4TileN;
    p.epoch = g_epoch.fetch_add(1);
    const long long tiles = static_cast<long long>(p.tiles_m) * p.tiles_n;
    if (tiles > 0x7FFFFFFFLL) return fail(SBSA_ERR_UNSUPPORTED, "too many tiles");
    const int grid = static_cast<int>(tiles < sm_count() ? tiles : sm_count());
    cudaError_t e = cudaFuncSetAttribute(nvfp4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFp4SmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "nvfp4 gemm smem attribute");
    nvfp4_gemm_kernel<<<grid, kFp4Threads, kFp4SmemBytes, static_cast<cudaStream_t>(stream)>>>(ma, mb, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "nvfp4 gemm launch");
    return ok();
}

sbsa_status sbsa_select_blocks(const sbsa_shape* shape, const float* q_mean, const float* k_mean, int32_t k_keep,
                               int32_t* row_ptr, int32_t* col_idx, void* stream) {
    sbsa_status r = check_shape(shape);
    if (r != SBSA_OK) return r;
    if ((r = check_k(shape, k_keep)) != SBSA_OK) return r;
    if (!q_mean || !k_mean || !row_ptr || !col_idx) return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(q_mean) || !aligned16(k_mean)) return fail(SBSA_ERR_INVALID_ARG, "means must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(row_ptr) | reinterpret_cast<uintptr_t>(col_idx)) & 3u)
        return fail(SBSA_ERR_INVALID_ARG, "row_ptr/col_idx must be 4-byte aligned");
    if ((r = launch_select(shape, q_mean, k_mean, k_keep, row_ptr, col_idx, static_cast<cudaStream_t>(stream))) !=
        SBSA_OK)
        return r;
    return ok();
}

sbsa_status sbsa_attention_fwd(const sbsa_shape* shape, const void* q, const void* k, const void* v,
                               const int32_t* row_ptr, const int32_t* col_idx, float scale, void* o, void* stream) {
    sbsa_status r = check_shape(shape);
    if (r != SBSA_OK) return r;
    if (!q || !k || !v || !o || !row_ptr || !col_idx) return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return fail(SBSA_ERR_INVALID_ARG, "q, k, v, o must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(row_ptr) | reinterpret_cast<uintptr_t>(col_idx)) & 3u)
        return fail(SBSA_ERR_INVALID_ARG, "row_ptr/col_idx must be 4-byte aligned");
    if (!std::isfinite(scale)) return fail(SBSA_ERR_INVALID_ARG, "scale must be finite");
    if ((r = launch_attn(shape, q, k, v, row_ptr, col_idx, resolve_scale(shape, scale), o,
                         static_cast<cudaStream_t>(stream))) != SBSA_OK)
        return r;
    return ok();
}

sbsa_status sbsa_forward(const sbsa_shape* shape, const void* q, const void* k, const void* v, int32_t k_keep,
                         float scale, void* o, int32_t* col_idx_out, void* workspace, size_t workspace_bytes,
                         void* stream) {
    sbsa_status r = check_shape(shape);
    if (r != SBSA_OK) return r;
    if ((r = check_k(shape, k_keep)) != SBSA_OK) return r;
    if (!q || !k || !v || !o) return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return fail(SBSA_ERR_INVALID_ARG, "q, k, v, o must be 16-byte aligned");
    if (col_idx_out && (reinterpret_cast<uintptr_t>(col_idx_out) & 3u))
        return fail(SBSA_ERR_INVALID_ARG, "col_idx_out must be 4-byte aligned");
    if (!std::isfinite(scale)) return fail(SBSA_ERR_INVALID_ARG, "scale must be finite");
    const WsLayout w = ws_layout(shape, k_keep);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return fail(SBSA_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
    if (workspace_bytes < w.total)
        return fail(SBSA_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed", workspace_bytes,
                    w.total);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* qm = reinterpret_cast<float*>(ws + w.q_mean);
    float* km = reinterpret_cast<float*>(ws + w.k_mean);
    int32_t* rp = reinterpret_cast<int32_t*>(ws + w.row_ptr);
    int32_t* ci = col_idx_out ? col_idx_out : reinterpret_cast<int32_t*>(ws + w.col_idx);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((r = launch_pool(shape, q, k, qm, km, st)) != SBSA_OK) return r;
    if ((r = launch_select(shape, qm, km, k_keep, rp, ci, st)) != SBSA_OK) return r;
    if ((r = launch_attn(shape, q, k, v, rp, ci, resolve_scale(shape, scale), o, st)) != SBSA_OK) return r;
    return ok();
}

sbsa_status sbsa_forward_host(const sbsa_shape* shape, const void* q_host, const void* k_host, const void* v_host,
                              int32_t k_keep, float scale, void* o_host, void* q, void* k, void* v, void* o,
                              void* workspace, size_t workspace_bytes, int32_t pairs_per_chunk, void* stream,
                              void* h2d_stream, void* d2h_stream) {
    sbsa_status r = check_shape(shape);
    if (r != SBSA_OK) return r;
    if ((r = check_k(shape, k_keep)) != SBSA_OK) return r;
    if (!q_host || !k_host || !v_host || !o_host) return fail(SBSA_ERR_INVALID_ARG, "null host pointer");
    if (!q || !k || !v || !o) return fail(SBSA_ERR_INVALID_ARG, "null device pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return fail(SBSA_ERR_INVALID_ARG, "q, k, v, o must be 16-byte aligned");
    if (!std::isfinite(scale)) return fail(SBSA_ERR_INVALID_ARG, "scale must be finite");
    if (pairs_per_chunk < 0) return fail(SBSA_ERR_INVALID_ARG, "pairs_per_chunk must be >= 0");
    const WsLayout w = ws_layout(shape, k_keep);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return fail(SBSA_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
    if (workspace_bytes < w.total)
        return fail(SBSA_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed", workspace_bytes,
                    w.total);
    const int pairs = shape->batch * shape->heads;
    const int n = pairs_per_chunk > 0 ? pairs_per_chunk : (pairs + 7) / 8;  // about eight chunks by default
    const size_t pair_bytes = static_cast<size_t>(shape->seq_len_padded) * shape->head_dim * 2;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaStream_t s_in = h2d_stream ? static_cast<cudaStream_t>(h2d_stream) : st;
    cudaStream_t s_out = d2h_stream ? static_cast<cudaStream_t>(d2h_stream) : st;
    cudaEvent_t ev[3] = {nullptr, nullptr, nullptr};  // start, copy-in done, chunk computed
    for (auto& e : ev) {
        cudaError_t ce = cudaEventCreateWithFlags(&e, cudaEventDisableTiming);
        if (ce != cudaSuccess) {
            for (auto& x : ev)
                if (x) cudaEventDestroy(x);
            return cuda_fail(ce, "event create");
        }
    }
    auto finish = [&](sbsa_status res) {
        for (auto& x : ev) cudaEventDestroy(x);  // released once their last record completes
        return res;
    };
    cudaError_t e;
    // the copies into q/k/v must wait for earlier work on `stream` that may still read them
    if ((e = cudaEventRecord(ev[0], st)) != cudaSuccess) return finish(cuda_fail(e, "event record"));
    if ((e = cudaStreamWaitEvent(s_in, ev[0], 0)) != cudaSuccess) return finish(cuda_fail(e, "stream wait"));
    if ((e = cudaStreamWaitEvent(s_out, ev[0], 0)) != cudaSuccess) return finish(cuda_fail(e, "stream wait"));
    const float sc = resolve_scale(shape, scale);
    for (int c0 = 0; c0 < pairs; c0 += n) {
        const int c1 = c0 + n < pairs ? c0 + n : pairs;
        const size_t off = static_cast<size_t>(c0) * pair_bytes, bytes = static_cast<size_t>(c1 - c0) * pair_bytes;
        // one copy per tensor and chunk (no batched-copy API)
        const void* src[3] = {q_host, k_host, v_host};
        void* dst[3] = {q, k, v};
        for (int t = 0; t < 3; ++t) {
            e = cudaMemcpyAsync(static_cast<uint8_t*>(dst[t]) + off, static_cast<const uint8_t*>(src[t]) + off, bytes,
                                cudaMemcpyHostToDevice, s_in);
            if (e != cudaSuccess) return finish(cuda_fail(e, "host-to-device copy"));
        }
        if ((e = cudaEventRecord(ev[1], s_in)) != cudaSuccess) return finish(cuda_fail(e, "event record"));
        if ((e = cudaStreamWaitEvent(st, ev[1], 0)) != cudaSuccess) return finish(cuda_fail(e, "stream wait"));
        // the chunk's (batch, head) pairs are a contiguous slab: one shape of c1 - c0 heads
        sbsa_shape cs = *shape;
        cs.batch = 1;
        cs.heads = c1 - c0;
        const WsLayout cw = ws_layout(&cs, k_keep);
        uint8_t* ws = static_cast<uint8_t*>(workspace);
        float* qm = reinterpret_cast<float*>(ws + cw.q_mean);
        float* km = reinterpret_cast<float*>(ws + cw.k_mean);
        int32_t* rp = reinterpret_cast<int32_t*>(ws + cw.row_ptr);
        int32_t* ci = reinterpret_cast<int32_t*>(ws + cw.col_idx);
        const uint8_t* cq = static_cast<const uint8_t*>(q) + off;
        const uint8_t* ck = static_cast<const uint8_t*>(k) + off;
        const uint8_t* cv = static_cast<const uint8_t*>(v) + off;
        uint8_t* co = static_cast<uint8_t*>(o) + off;
        if ((r = launch_pool(&cs, cq, ck, qm, km, st)) != SBSA_OK) return finish(r);
        if ((r = launch_select(&cs, qm, km, k_keep, rp, ci, st)) != SBSA_OK) return finish(r);
        if ((r = launch_attn(&cs, cq, ck, cv, rp, ci, sc, co, st)) != SBSA_OK) return finish(r);
        if ((e = cudaEventRecord(ev[2], st)) != cudaSuccess) return finish(cuda_fail(e, "event record"));
        if ((e = cudaStreamWaitEvent(s_out, ev[2], 0)) != cudaSuccess) return finish(cuda_fail(e, "stream wait"));
        e = cudaMemcpyAsync(static_cast<uint8_t*>(o_host) + off, co, bytes, cudaMemcpyDeviceToHost, s_out);
        if (e != cudaSuccess) return finish(cuda_fail(e, "device-to-host copy"));
    }
    // the caller's stream completes only after the last copy-out
    if ((e = cudaEventRecord(ev[0], s_out)) != cudaSuccess) return finish(cuda_fail(e, "event record"));
    if ((e = cudaStreamWaitEvent(st, ev[0], 0)) != cudaSuccess) return finish(cuda_fail(e, "stream wait"));
    return finish(ok());
}

sbsa_status sbsa_forward_noalloc(const sbsa_shape* shape, const void* q, const void* k, const void* v,
                                 int32_t k_keep, float scale, void* o, int32_t* col_idx_out, void* stream) {
    sbsa_status r = check_shape(shape);
    if (r != SBSA_OK) return r;
    if ((r = check_k(shape, k_keep)) != SBSA_OK) return r;
    if (!q || !k || !v || !o) return fail(SBSA_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return fail(SBSA_ERR_INVALID_ARG, "q, k, v, o must be 16-byte aligned");
    if (col_idx_out && (reinterpret_cast<uintptr_t>(col_idx_out) & 3u))
        return fail(SBSA_ERR_INVALID_ARG, "col_idx_out must be 4-byte aligned");
    if (!std::isfinite(scale)) return fail(SBSA_ERR_INVALID_ARG, "scale must be finite");
    const WsLayout w = ws_layout(shape, k_keep);
    if (w.total > kNoAllocScratchBytes)
        return fail(SBSA_ERR_WORKSPACE,
                    "this shape needs %zu bytes of scratch; the built-in scratch holds %zu (use sbsa_forward "
                    "with a workspace)",
                    w.total, kNoAllocScratchBytes);
    void* scratch = nullptr;
    if ((r = noalloc_scratch(&scratch)) != SBSA_OK) return r;
    uint8_t* ws = static_cast<uint8_t*>(scratch);
    float* qm = reinterpret_cast<float*>(ws + w.q_mean);
    float* km = reinterpret_cast<float*>(ws + w.k_mean);
    int32_t* rp = reinterpret_cast<int32_t*>(ws + w.row_ptr);
    int32_t* ci = col_idx_out ? col_idx_out : reinterpret_cast<int32_t*>(ws + w.col_idx);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // every scratch element the later kernels read is written earlier in this call,
    // so nothing needs clearing between calls
    if ((r = launch_pool(shape, q, k, qm, km, st)) != SBSA_OK) return r;
    if ((r = launch_select(shape, qm, km, k_keep, rp, ci, st)) != SBSA_OK) return r;
    if ((r = launch_attn(shape, q, k, v, rp, ci, resolve_scale(shape, scale), o, st)) != SBSA_OK) return r;
    return ok();
}

sbsa_status sbsa_set_pipeline_wait_ns(uint64_t limit_ns) {
    const unsigned long long v = limit_ns;
    cudaError_t e = cudaMemcpyToSymbol(g_pipe_wait_ns, &v, sizeof v);
    if (e != cudaSuccess) return cuda_fail(e, "set pipeline wait limit");
    return ok();
}

sbsa_status sbsa_check(void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    unsigned int bits = 0, zero = 0;
    if ((e = cudaMemcpyFromSymbol(&bits, g_error_bits, sizeof bits)) != cudaSuccess)
        return cuda_fail(e, "read error word");
    if ((e = cudaMemcpyToSymbol(g_error_bits, &zero, sizeof zero)) != cudaSuccess)
        return cuda_fail(e, "clear error word");
    if (bits & kErrTimeout) return fail(SBSA_ERR_TIMEOUT, "a kernel wait ran out of time");
    if (bits & kErrBadIndex) return fail(SBSA_ERR_BAD_INDEX, "a block index or row pointer was out of range");
    return ok();
}

sbsa_status sbsa_validate_csr(const sbsa_shape* shape, const int32_t* row_ptr, const int32_t* col_idx, int64_t nnz,
                              int32_t require_diagonal, void* stream) {
    sbsa_status r = check_shape(shape);
    if (r != SBSA_OK) return r;
    if (!row_ptr || (!col_idx && nnz > 0) || nnz < 0) return fail(SBSA_ERR_INVALID_ARG, "null pointer or nnz < 0");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned int* bad = nullptr;  // module-scope device flag (no allocation)
    cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&bad), g_csr_bad);
    if (e != cudaSuccess) return cuda_fail(e, "csr flag address");
    if ((e = cudaMemsetAsync(bad, 0, sizeof(unsigned int), st)) != cudaSuccess) return cuda_fail(e, "csr flag clear");
    const long long nrows = num_rows(shape);
    const long long threads = nrows + 1;
    validate_csr_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, st>>>(
        row_ptr, col_idx, nrows, nnz, num_blocks(shape), require_diagonal, bad);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "csr validate launch");
    unsigned int h = 0;
    if ((e = cudaMemcpyAsync(&h, bad, sizeof h, cudaMemcpyDeviceToHost, st)) != cudaSuccess)
        return cuda_fail(e, "csr flag read");
    if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(e, "stream synchronize");
    if (h) return fail(SBSA_ERR_BAD_INDEX, "CSR block list is malformed");
    return ok();
}

}  // extern "C"
