/*
 * sbsa -- dynamic block-sparse self-attention for NVIDIA B200 (sm_100a).
 *
 * The method (the hot path of 14B video-DiT inference at ~120K tokens):
 *   1. pool   : block-level means of Query and Key estimate attention importance
 *               (page "知识卡片：600倍加速，720p视频实时生成！单卡也能带的动14B模型",
 *               section 方法/产品要点, bullet 动态稀疏量化注意力);
 *   2. select : each query block keeps only ~10-20% of the key blocks, decided at run
 *               time per input (same bullet, "稀疏率 80%-90%");
 *   3. attend : the kept blocks are computed densely
 *               (page "单卡 RTX 5090 跑 Wan2.2-A14B：720p 视频生成只要 3.8 秒",
 *               section 四步拆解, item 3 动态稀疏注意力).
 *
 * Readings this library takes where those pages are silent: the score of a (query
 * block i, key block j) pair is <qmean_i, kmean_j>; each query block keeps a fixed
 * count k of key blocks, the diagonal j == i always among them, the rest the k-1
 * highest scores, ties to the lower block index; attention is non-causal with scale
 * 1/sqrt(d) by default; padded tokens are masked as keys and produce zero rows.
 *
 * Conventions for every entry point:
 *   - Tensors are row-major, contiguous [B][H][Lp][d] (bf16 for Q/K/V/O), block means
 *     [B][H][nb][d] fp32, where nb = Lp / block_size.  Device pointers.  bf16 and fp32
 *     tensors must be 16-byte aligned.
 *   - The caller owns every buffer.  No call allocates device memory.
 *   - All calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL is
 *     the legacy default stream).  Argument errors are returned before anything is
 *     launched.  Errors detected on the device (a bounded wait that ran out, an
 *     out-of-range block index) are latched in a per-device error word and reported by
 *     sbsa_check().
 *   - Calls are safe to issue from several host threads; the last error message is
 *     thread-local.
 */
#ifndef SBSA_H
#define SBSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SBSA_OK = 0,
    SBSA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, inconsistent shape, k out of range */
    SBSA_ERR_UNSUPPORTED = 2, /* head_dim or block_size not in {64,128}, too many blocks */
    SBSA_ERR_WORKSPACE = 3,   /* workspace missing, misaligned or smaller than sbsa_workspace_bytes() */
    SBSA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed (launch, tensor-map encode) */
    SBSA_ERR_TIMEOUT = 5,     /* a kernel's bounded wait expired (device-side, via sbsa_check) */
    SBSA_ERR_BAD_INDEX = 6    /* a CSR block index / row pointer was out of range (device-side) */
} sbsa_status;

/* Problem shape.  seq_len = L valid tokens; seq_len_padded = Lp must be the smallest
 * multiple of block_size >= L (every block holds at least one valid token).
 * head_dim in {64, 128}; block_size in {64, 128}; nb = Lp / block_size <= 2048;
 * batch * heads * Lp < 2^31. */
typedef struct {
    int32_t batch;
    int32_t heads;
    int32_t seq_len;
    int32_t seq_len_padded;
    int32_t head_dim;
    int32_t block_size;
} sbsa_shape;

/* Library version, major*10000 + minor*100 + patch. */
int32_t sbsa_version(void);

/* Human-readable name of a status code (static string). */
const char *sbsa_status_string(sbsa_status status);

/* Detail of the last error returned on the calling host thread ("" if none). */
const char *sbsa_last_error_message(void);

/* Kept key blocks per query block for a keep fraction: round-half-up(keep * nb),
 * clamped to [1, nb].  ("keep about 10-20% of the blocks" read as a per-row count.)
 * Returns 0 if num_blocks < 1 or keep_fraction is not finite. */
int32_t sbsa_keep_blocks(int32_t num_blocks, double keep_fraction);

/* Bytes of workspace sbsa_forward() needs: q_mean and k_mean (fp32, B*H*nb*d each),
 * row_ptr (int32, B*H*nb+1) and col_idx (int32, B*H*nb*k), each 256-byte aligned.
 * Returns 0 for an invalid shape or k. */
size_t sbsa_workspace_bytes(const sbsa_shape *shape, int32_t k_keep);

/* Step 1 -- block means (page "知识卡片…", 方法/产品要点, 动态稀疏量化注意力: Q/K
 * block-level means as the importance estimate).
 *   q, k   : bf16 [B][H][Lp][d] (device).  Padded tokens may hold any value.
 *   q_mean : fp32 [B][H][nb][d] (device, written) = mean of Q over the valid tokens
 *            of each block; k_mean likewise for K.
 * One kernel launch, HBM-bandwidth bound. */
sbsa_status sbsa_pool_qk(const sbsa_shape *shape, const void *q, const void *k, float *q_mean, float *k_mean,
                         void *stream);

/* Step 0 fused with step 1 -- 3D RoPE of Q and K, then their block means (pages
 * "知识卡片…", 方法/产品要点, bullet 高效推理算子, and "单卡 RTX 5090 跑 Wan2.2-A14B…",
 * 四步拆解 item 4: 3D RoPE as a fused kernel, fewer temporaries and memory round trips;
 * here it is fused with the pooling that follows, so Q and K cross HBM once for both).
 * The pages give no frequencies.  The rotation used: the head dimension is cut into
 * pairs (2p, 2p+1); the first P_T = d/2 - 2*P_H pairs turn with the token's frame
 * index, the next P_H = floor(d/6) with its row index, the last P_W = P_H with its
 * column index on the (grid_t, grid_h, grid_w) latent grid, tokens in row-major order
 * (d = 128: 22 + 21 + 21 pairs; d = 64: 12 + 10 + 10); pair q of an axis with P pairs
 * turns by pos * theta^(-q/P):  (x, y) -> (x cos - y sin, x sin + y cos).
 *
 * sbsa_rope_table_floats: floats of the cos/sin table for a grid (0 if invalid).
 * sbsa_rope_table_init: fills `table` (device, 8-byte aligned, that many floats) with
 *   (cos, sin) pairs computed in double and rounded to fp32; theta > 1 (10000 usual).
 *   One small launch; the table can be kept for every layer with the same grid.
 * sbsa_rope_pool_qk: grid_t * grid_h * grid_w must equal seq_len.
 *   q, k         : bf16 [B][H][Lp][d] (device) before the rotation.
 *   q_out, k_out : bf16 [B][H][Lp][d] (device, written): rotated in fp32, rounded to
 *                  bf16 (ties to even).  May be the same buffers as q, k (in place).
 *                  Padded tokens t >= L are copied unrotated.
 *   q_mean, k_mean: fp32 [B][H][nb][d] (device, written): means of the rotated bf16
 *                  values over the valid tokens of each block, as sbsa_pool_qk of q_out
 *                  and k_out would give.
 * One kernel launch, HBM-bandwidth bound (reads Q and K once, writes them once). */
size_t sbsa_rope_table_floats(int32_t head_dim, int32_t grid_t, int32_t grid_h, int32_t grid_w);
sbsa_status sbsa_rope_table_init(int32_t head_dim, int32_t grid_t, int32_t grid_h, int32_t grid_w, double theta,
                                 float *table, void *stream);
sbsa_status sbsa_rope_pool_qk(const sbsa_shape *shape, int32_t grid_t, int32_t grid_h, int32_t grid_w,
                              const float *table, const void *q, const void *k, void *q_out, void *k_out,
                              float *q_mean, float *k_mean, void *stream);

/* Step 2 -- block selection (same bullet: keep ~10-20% of the blocks, chosen per
 * input at run time).  For each (b, h, query block i): score_j = <q_mean_i, k_mean_j>
 * in fp32; keep j = i plus the k_keep-1 highest-scoring other blocks (ties: lower j);
 * write them in ascending order.
 *   q_mean, k_mean : fp32 [B][H][nb][d] (device).  Scores must be finite.
 *   k_keep         : 1 <= k_keep <= nb.
 *   row_ptr        : int32 [B*H*nb + 1] (device, written) CSR row offsets, r * k_keep.
 *   col_idx        : int32 [B*H*nb*k_keep] (device, written) key-block indices.
 * One kernel launch. */
sbsa_status sbsa_select_blocks(const sbsa_shape *shape, const float *q_mean, const float *k_mean, int32_t k_keep,
                               int32_t *row_ptr, int32_t *col_idx, void *stream);

/* Step 3 -- dense attention inside the kept blocks (page "单卡 RTX 5090 跑
 * Wan2.2-A14B…", 四步拆解 item 3: kept blocks computed densely).  For every valid query
 * row t of query block i:  O[t] = sum over valid keys u of the blocks listed in
 * col_idx[row_ptr[r] .. row_ptr[r+1]) of softmax_u(scale * Q[t].K[u]) V[u], where
 * r = (b*H + h)*nb + i.  Non-causal.  Rows t >= L, and rows whose list holds no valid
 * key, are written as 0.
 *   q, k, v : bf16 [B][H][Lp][d] (device).
 *   row_ptr : int32 [B*H*nb + 1], non-decreasing, row_ptr[0] == 0; any list length.
 *   col_idx : int32 key-block indices in [0, nb), in any order; a block listed twice
 *             contributes its keys twice.  An index outside that range is skipped
 *             (contributes nothing) and latches SBSA_ERR_BAD_INDEX.
 *   scale   : logit scale; 0 means 1/sqrt(head_dim).
 *   o       : bf16 [B][H][Lp][d] (device, written).
 * Arithmetic: bf16 tensor-core products (tcgen05) with fp32 accumulation, fp32 online
 * softmax, probabilities rounded to bf16 before the P.V product, bf16 output. */
sbsa_status sbsa_attention_fwd(const sbsa_shape *shape, const void *q, const void *k, const void *v,
                               const int32_t *row_ptr, const int32_t *col_idx, float scale, void *o, void *stream);

/* The FP8 path (pages "知识卡片…", 方法/产品要点, bullet 动态稀疏量化注意力, and "单卡 RTX
 * 5090 跑 Wan2.2-A14B…", 四步拆解 item 3: the sparse mask feeds an FP8 attention in the
 * style of SageAttention2).  The pages give no quantization detail; what is built:
 * K smoothed by its sequence mean (softmax is unchanged by subtracting one vector from
 * every key), one scale per block of Q and of K, e4m3 codes, S = Q.K^T on e4m3 tensor
 * cores with fp32 accumulation, and the rest (softmax, P.V in bf16) as in step 3.
 * head_dim 128 only.
 *
 * sbsa_key_mean: out fp32 [B][H][d] (device, written) = sum over blocks of
 *   (valid tokens of the block) * k_mean[b,h,block,:] / L, i.e. the mean of K over the
 *   valid tokens, from the block means of sbsa_pool_qk.
 * sbsa_quantize_qk_fp8: q, k bf16 [B][H][Lp][d]; k_smooth fp32 [B][H][d] or NULL (no
 *   smoothing); q8, k8 uint8 [B][H][Lp][d] (device, written) e4m3 codes; q_scale,
 *   k_scale fp32 [B][H][nb] (device, written).  Per block, in fp32: y = x - smooth (K
 *   only), amax = max |y| over the valid tokens, code = e4m3(y * (448 / amax)) with
 *   round-to-nearest-even and saturation at +-448, scale = amax / 448 (1 for an all-zero
 *   block); padded tokens get code 0.  One launch, HBM-bandwidth bound.
 * sbsa_attention_fwd_fp8: as sbsa_attention_fwd, with q8/k8 and their block scales in
 *   place of q/k: the logits are scale * (q8 . k8) * q_scale[query block] *
 *   k_scale[key block].  v and o are bf16 as before. */
sbsa_status sbsa_key_mean(const sbsa_shape *shape, const float *k_mean, float *out, void *stream);
sbsa_status sbsa_quantize_qk_fp8(const sbsa_shape *shape, const void *q, const void *k, const float *k_smooth,
                                 void *q8, void *k8, float *q_scale, float *k_scale, void *stream);
sbsa_status sbsa_attention_fwd_fp8(const sbsa_shape *shape, const void *q8, const void *k8, const void *v,
                                   const float *q_scale, const float *k_scale, const int32_t *row_ptr,
                                   const int32_t *col_idx, float scale, void *o, void *stream);

/* ---- NVFP4 linear layers (the GEMMs around the attention) ---------------------------
 * Page "知识卡片：600倍加速，720p视频实时生成！单卡也能带的动14B模型", 方法/产品要点, bullets
 * NVFP4 量化感知训练 (E2M1 values, one FP8 scale per 16 consecutive elements, an FP32
 * scale per tensor) and 高效推理算子 (both GEMM operands NVFP4 on the block-scaled tensor
 * cores); page "单卡 RTX 5090 跑 Wan2.2-A14B：720p 视频生成只要 3.8 秒", 四步拆解 item 2
 * (FP32 accumulation, BF16 output, column bias fused into the epilogue).
 *
 * Formats (the pages give no formula; this is the reading taken):
 *   tensor scale s = 2688 / amax|x| (1 for an all-zero tensor), 2688 = 6 * 448;
 *   block scale sf = e4m3((amax of the 16 elements / 6) * s), round to nearest even,
 *   saturating; code = e2m1(x * (s / sf)), nearest even, saturating at +-6 (0 where
 *   sf = 0); all in fp32, in this order.  Value = e2m1(code) * e4m3(sf) / s.
 *   codes:  [rows][cols/2] bytes, row-major; element 2i of a row in the low nibble of
 *           byte i.
 *   scales: sbsa_nvfp4_scale_bytes(rows, cols) bytes; atoms of 128 rows x 4 blocks (512
 *           bytes: row r at (r % 32) * 16 + ((r % 128) / 32) * 4, block kb at + kb % 4),
 *           the cols/64 atoms of one 128-row group consecutive, groups in row order;
 *           rows past the matrix (up to a multiple of 128) have scale 0.
 * All pointers are device pointers owned by the caller; every call is asynchronous on
 * `stream`; argument errors are returned before any launch, launch errors as
 * SBSA_ERR_CUDA, and a kernel that gives up on a wait latches SBSA_ERR_TIMEOUT for
 * sbsa_check.
 *
 * sbsa_nvfp4_scale_bytes: size of the scale array of a [rows][cols] matrix (cols a
 *   multiple of 64), 0 for invalid sizes.
 * sbsa_nvfp4_amax: *amax = max |x| over a bf16 [rows][cols] matrix (16-byte aligned,
 *   cols a multiple of 8).  Resets *amax first, then one reduction launch.
 * sbsa_nvfp4_quantize: bf16 [rows][cols] (cols a multiple of 64) -> codes and scales,
 *   with the tensor scale taken from *amax (device, as written by sbsa_nvfp4_amax).
 * sbsa_nvfp4_gemm: c[m][n] (bf16, row-major) = A B^T / (s_A s_B) + bias[n], A = [m][k]
 *   and B = [n][k] as NVFP4 codes + scales, s_A and s_B from a_amax / b_amax (device).
 *   bias ([n] fp32) may be NULL.  Needs k a multiple of 256, n a multiple of 8; m any.
 *   Codes, scales and c 16-byte aligned. */
size_t sbsa_nvfp4_scale_bytes(int64_t rows, int32_t cols);
sbsa_status sbsa_nvfp4_amax(const void *x, int64_t rows, int32_t cols, float *amax, void *stream);
sbsa_status sbsa_nvfp4_quantize(const void *x, int64_t rows, int32_t cols, const float *amax, void *codes,
                                void *scales, void *stream);
sbsa_status sbsa_nvfp4_gemm(int32_t m, int32_t n, int32_t k, const void *a, const void *a_scales, const float *a_amax,
                            const void *b, const void *b_scales, const float *b_amax, const float *bias, void *c,
                            void *stream);

/* ---- Light-Ulysses sequence parallelism ------------------------------------------------
 * Page "知识卡片：600倍加速，720p视频实时生成！单卡也能带的动14B模型", 方法/产品要点, bullet
 * Light-Ulysses 多卡并行; page "单卡 RTX 5090 跑 Wan2.2-A14B：720p 视频生成只要 3.8 秒",
 * 四步拆解 item 4: Ulysses-style sequence parallelism with an FP8 payload, Q, K and V fused
 * into one all-to-all, fused pre/post-processing kernels and a head-level pipeline.
 * These calls are the pre/post-processing around the caller's all-to-all (NCCL), or, with
 * the peer-put calls below, the exchange itself.
 *
 * `world` ranks; before the attention rank r holds tokens [r L/world, (r+1) L/world), during
 * it heads [r H/world, (r+1) H/world).  A head chunk (head0, head_chunk) selects heads
 * head0 .. head0 + head_chunk - 1 of every rank's H/world (one step of the head-level
 * pipeline; head0 = 0, head_chunk = H/world for the whole exchange).  Every row of
 * head_dim = 128 values crosses as 128 e4m3 codes and one fp32 scale: scale = amax/448,
 * code = e4m3(x * (448/amax)) in fp32, nearest even, saturating (an all-zero row: scale 1,
 * codes 0); the receiver restores bf16(code * scale).
 *
 * Buffers: `send`/`recv` hold `world` equal slices in rank order, each slice its codes then
 * its scales, padded to a multiple of 16 bytes.  QKV slice for peer j: codes [L/world][3][head_chunk][128], scales
 * [L/world][3][head_chunk] (fp32); O slice: codes [L/world][head_chunk][128], scales
 * [L/world][head_chunk].  The all-to-all sends slice j of `send` to rank j and writes the
 * slice from rank i at slice i of `recv`.
 *   x: [L/world][3][H][128] bf16 (the fused QKV activation of this rank's tokens)
 *   q, k, v, o: [H/world][tokens_padded][128] bf16 (the attention layout; unpack writes
 *     the chunk's heads, tokens >= L as zero)
 *   y: [L/world][H][128] bf16 (every head of this rank's tokens)
 * Device pointers owned by the caller, 16-byte aligned; asynchronous on `stream`;
 * argument errors before any launch.  *_bytes return 0 for invalid arguments. */
typedef struct {
    int32_t world;          /* ranks G */
    int32_t tokens;         /* L, a multiple of world */
    int32_t tokens_padded;  /* rows of the attention layout, >= L */
    int32_t heads;          /* H, a multiple of world */
    int32_t head_dim;       /* 128 */
} sbsa_ulysses_shape;

size_t sbsa_ulysses_qkv_bytes(const sbsa_ulysses_shape *shape, int32_t head_chunk);
size_t sbsa_ulysses_o_bytes(const sbsa_ulysses_shape *shape, int32_t head_chunk);
sbsa_status sbsa_ulysses_pack_qkv(const sbsa_ulysses_shape *shape, int32_t head0, int32_t head_chunk, const void *x,
                                  void *send, void *stream);
sbsa_status sbsa_ulysses_unpack_qkv(const sbsa_ulysses_shape *shape, int32_t head0, int32_t head_chunk,
                                    const void *recv, void *q, void *k, void *v, void *stream);
sbsa_status sbsa_ulysses_pack_o(const sbsa_ulysses_shape *shape, int32_t head0, int32_t head_chunk, const void *o,
                                void *send, void *stream);
sbsa_status sbsa_ulysses_unpack_o(const sbsa_ulysses_shape *shape, int32_t head0, int32_t head_chunk,
                                  const void *recv, void *y, void *stream);

/* Peer-put exchange: the same slices, written by the packing kernel straight into every
 * peer's receive buffer (peer-mapped memory over NVLink) instead of a send buffer and a
 * collective.  Each rank's exchange allocation (the same layout on every rank) holds the
 * receive buffers and arrays of uint32 flags.
 *   peer_bases: device array of `world` uint64 base addresses of the ranks' allocations,
 *     as mapped in this process (peer_bases[rank] is this rank's own); 16-byte aligned.
 *   recv_offset: byte offset of the receive buffer inside each allocation (multiple of 16).
 *     Slice `rank` of peer j's receive buffer gets this rank's rows for peer j.
 * sbsa_ulysses_put_qkv / sbsa_ulysses_put_o: pack as sbsa_ulysses_pack_qkv / _pack_o, the
 *   slice for peer j written at peer_bases[j] + recv_offset + rank * slice bytes; the
 *   stores are visible system-wide when the launch ends.
 * sbsa_peer_signal: flag word `rank` of the uint32 array at flag_offset (a multiple of 4)
 *   in every peer's allocation := value, a system-scope release ordered after the
 *   stream's earlier launches.
 * sbsa_peer_wait: waits on the device until flags[0 .. world) all equal value
 *   (system-scope acquire), then the stream's later launches run; after timeout_s seconds
 *   (0 < timeout_s <= 60) it gives up and latches SBSA_ERR_TIMEOUT for sbsa_check (no
 *   fault, no hang).  world is at most 1024 here and in sbsa_peer_signal.
 * Values are the caller's (an epoch per exchange and buffer, so no stale flag matches).
 * The contents of peer_bases cannot be checked on the host: every entry must map a live
 * allocation of the layout above. */
sbsa_status sbsa_ulysses_put_qkv(const sbsa_ulysses_shape *shape, int32_t head0, int32_t head_chunk, const void *x,
                                 const uint64_t *peer_bases, uint64_t recv_offset, int32_t rank, void *stream);
sbsa_status sbsa_ulysses_put_o(const sbsa_ulysses_shape *shape, int32_t head0, int32_t head_chunk, const void *o,
                               const uint64_t *peer_bases, uint64_t recv_offset, int32_t rank, void *stream);
sbsa_status sbsa_peer_signal(const uint64_t *peer_bases, uint64_t flag_offset, int32_t rank, int32_t world,
                             uint32_t value, void *stream);
sbsa_status sbsa_peer_wait(const uint32_t *flags, int32_t world, uint32_t value, double timeout_s, void *stream);

/* Steps 1-3 in one call on one stream: pool -> select -> attend, with the means and
 * the CSR lists carved out of `workspace` (device, 256-byte aligned, at least
 * sbsa_workspace_bytes(shape, k_keep) bytes).  If col_idx_out is non-NULL the
 * selected blocks ([B*H*nb*k_keep] int32, device) are written there as well. */
sbsa_status sbsa_forward(const sbsa_shape *shape, const void *q, const void *k, const void *v, int32_t k_keep,
                         float scale, void *o, int32_t *col_idx_out, void *workspace, size_t workspace_bytes,
                         void *stream);

/* Steps 1-3 end to end from host memory (page "单卡 RTX 5090 跑 Wan2.2-A14B：720p 视频
 * 生成只要 3.8 秒", section 四步拆解, item 3, computed as sbsa_forward does): copies Q, K, V
 * from the host into the device buffers q, k, v, runs pool -> select -> attend, and
 * copies O from the device buffer o back to o_host.
 *   q_host, k_host, v_host, o_host: HOST memory, [B][H][Lp][d] bf16 (Lp rows per
 *   (batch, head), padded rows included).  Pinned (page-locked) memory is what lets the
 *   copies run asynchronously and overlap the kernels; pageable memory gives the same
 *   result with copies the driver stages.  q, k, v, o: device buffers of the same size,
 *   16-byte aligned; workspace as for sbsa_forward (the full shape's size).
 *   The (batch, head) pairs are independent, so the call processes them in chunks of
 *   pairs_per_chunk pairs (0: about eight chunks): the copy-in of a chunk on h2d_stream,
 *   its three kernels on `stream` and its copy-out on d2h_stream, with events between the
 *   streams, so that copies of one chunk overlap the kernels of its neighbours.  One
 *   cudaMemcpyAsync per tensor and chunk.  The result equals one sbsa_forward call on the
 *   whole shape bit for bit.  h2d_stream / d2h_stream may be NULL (then `stream` does
 *   the copies too, without overlap); one stream for both copy directions is correct but
 *   serializes each copy-out with the next copy-in.
 *   Asynchronous: the work, copies included, is complete when `stream` is (the call makes
 *   `stream` wait for the last copy-out, and the first copy-in wait for work already
 *   queued on `stream`).  Host and device buffers must stay valid until then.  Creates
 *   and releases three CUDA events per call; allocates no memory.  On an error returned
 *   part way, the work already queued still runs; the returned status says what failed. */
sbsa_status sbsa_forward_host(const sbsa_shape *shape, const void *q_host, const void *k_host, const void *v_host,
                              int32_t k_keep, float scale, void *o_host, void *q, void *k, void *v, void *o,
                              void *workspace, size_t workspace_bytes, int32_t pairs_per_chunk, void *stream,
                              void *h2d_stream, void *d2h_stream);

/* sbsa_forward without a workspace, for callers that cannot allocate device memory:
 * for example a plug-in inside another engine that owns every device allocation, or
 * a latency-critical loop where cudaMalloc/cudaFree would synchronize the device.
 * The pages describe no such call; it exists only for these callers.
 *   Same arguments, results and launches as sbsa_forward, minus the workspace.  The
 *   block means and the CSR list go to a 16 MiB scratch array that the library
 *   reserves on every GPU it is loaded on, for the life of the process.  Shapes
 *   with sbsa_workspace_bytes(shape, k_keep) > 16 MiB (16,777,216 bytes) are rejected
 *   with SBSA_ERR_WORKSPACE before anything is launched.  Example: the 480p case
 *   (40 heads, 256 blocks of 128, d = 128, k = 51) needs 12.6 MB.
 *   Every call looks up the scratch array's device address in the current context
 *   (cudaGetSymbolAddress: a lookup, not an allocation), so the address stays valid
 *   after a device reset or a context switch.  The first call on a device may load
 *   the library's device code; make that first call before any stream capture.
 *   All calls share the one array, and it keeps the last call's contents.  Calls
 *   whose work overlaps on the GPU (different streams, or different host threads
 *   without ordering) race on it and must be serialized by the caller.  Every scratch
 *   element read within a call is written earlier in the same call, so nothing needs
 *   clearing.  This call allocates nothing: no cudaMalloc, no cudaFree, no allocating
 *   library routine. */
sbsa_status sbsa_forward_noalloc(const sbsa_shape *shape, const void *q, const void *k, const void *v,
                                 int32_t k_keep, float scale, void *o, int32_t *col_idx_out, void *stream);

/* Failure handling (a bounded wait in every kernel pipeline, latched as
 * SBSA_ERR_TIMEOUT; nothing traps): sets, on the current device, the limit of the
 * pipeline waits of the attention, selection, RoPE + pooling and FP8 quantizer kernels
 * launched afterwards.  Default 1e9 ns (1 s), far above any legitimate wait.  0 makes a
 * pipeline wait give up unless its barrier has already completed when first tested: a
 * test uses it to drive the give-up path (latch the error, make the launch's other CTAs
 * stop, wait for this CTA's own copies and tensor-core work, release its tensor memory)
 * without stalling a pipeline.  The waits of that drain keep their own 1 s limit.  The
 * NVFP4 GEMM keeps its fixed 1 s limit.  Synchronous; not for use while kernels of this
 * library run on the device. */
sbsa_status sbsa_set_pipeline_wait_ns(uint64_t limit_ns);

/* Synchronizes `stream`, then reads and clears the calling device's error word.
 * Returns SBSA_OK, SBSA_ERR_TIMEOUT, SBSA_ERR_BAD_INDEX or SBSA_ERR_CUDA (a sticky
 * CUDA error or a failed synchronize). */
sbsa_status sbsa_check(void *stream);

/* Validates a CSR block list on the device: row_ptr[0] == 0, non-decreasing,
 * row_ptr[nrows] == nnz, every index in [0, nb) and strictly ascending within a row,
 * and (if require_diagonal) each row r contains its own block r % nb.
 * Synchronous: it synchronizes `stream` and returns SBSA_OK or SBSA_ERR_BAD_INDEX. */
sbsa_status sbsa_validate_csr(const sbsa_shape *shape, const int32_t *row_ptr, const int32_t *col_idx, int64_t nnz,
                              int32_t require_diagonal, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SBSA_H */
