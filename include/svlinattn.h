/*
 * svlinattn — ReLU-kernel linear attention on NVIDIA B200 (sm_100a), C ABI.
 *
 * The operation (SANA-Video, "Efficient Video Generation with Block Linear Diffusion
 * Transformer"; talk at ICLR 2026, block KV cache passage, and the paper abstract, design (2)
 * "Constant-Memory KV cache for Block Linear Attention"):
 *
 *     phi(x) = max(x, 0)                                  (feature map, elementwise)
 *     S      = sum_j phi(k_j)^T v_j    [D x D]            (state: row = key feature d,
 *     z      = sum_j phi(k_j)          [D]                         column = value feature e)
 *     o_i    = phi(q_i) S / (phi(q_i) . z + eps)
 *
 * Linear attention keeps a state of fixed shape D x D whatever the sequence length. In the
 * block-causal form a video is generated block by block: a block attends to itself
 * (bidirectionally, it is diffused as a whole) and to the state summed over all previous blocks;
 * after the block, its own state is added to that cache. The cache (S, z) therefore has constant
 * size, B*H*D*(D+1) fp32 values, however many blocks have been generated.
 *
 * Conventions shared by every entry point
 *  - q, k, v, o are DEVICE pointers to contiguous [B, H, N, D] tensors (row-major, D fastest),
 *    element type `dt` (SV_BF16: bfloat16, SV_F32: float). o has the type of q. 16-byte aligned.
 *  - S is a DEVICE pointer to fp32 [B, H, D, D] (S[b][h][d][e], d = key feature, e = value
 *    feature), z a DEVICE pointer to fp32 [B, H, D]. 4-byte aligned. The cache is always fp32.
 *  - ws is caller-owned DEVICE scratch of at least sv_workspace_bytes(...) bytes, 256-byte
 *    aligned, zero-initialised once with sv_workspace_init before its first use. Its first
 *    256 bytes hold a status word that the kernels raise when a bounded wait expires.
 *    Calls that share one workspace must be ordered on the GPU (same stream, or synchronised).
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 *    Pointers stay owned by the caller; the library allocates nothing and keeps no state
 *    between calls other than per-device kernel attributes, with one exception: the library
 *    holds a static 16 MiB device array on every device that loads it, the scratch of
 *    sv_cache_step_noalloc, whose contents (status word, launch sequence number, flags) persist
 *    from one call of that entry point to the next.
 *  - Supported sizes: B, H, N >= 1; SV_BF16: D a multiple of 8 in [8, 128] (a row must be a whole
 *    number of 16-byte units); SV_F32: 1 <= D <= 128. eps must be finite and >= 0.
 *  - Errors: every argument is checked on the host BEFORE anything is launched; a bad argument
 *    returns SV_ERR_INVALID_ARG / SV_ERR_UNSUPPORTED and launches nothing. A failed launch returns
 *    SV_ERR_CUDA. Device-side timeouts (SV_ERR_TIMEOUT) are reported by sv_device_status.
 *    sv_last_error() gives a message for the calling thread's last non-OK status.
 *  - NaN/Inf inputs propagate; nothing checks for them.
 *  - Residency: with bf16 I/O and one block per head (sv_linattn_fwd, sv_cache_step and
 *    sv_block_causal_attn with block_len >= N) the work runs as one launch whose CTAs (one per SM
 *    at most) wait on one another, so they must all be resident together. On a device that other
 *    streams do not occupy this always holds. The launch overlaps its setup with the previous
 *    kernel (programmatic dependent launch); setting SV_FUSED_COOPERATIVE=1 in the environment
 *    makes it a cooperative launch instead, which the runtime only starts once every CTA fits.
 *    A CTA kept off the device for longer than the wait limit (2 s) makes the call report
 *    SV_ERR_TIMEOUT through sv_device_status; it never hangs.
 */
#ifndef SVLINATTN_H
#define SVLINATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SV_OK = 0,
  SV_ERR_INVALID_ARG = 1, /* null/misaligned pointer, size <= 0, workspace too small, bad eps */
  SV_ERR_UNSUPPORTED = 2, /* D or dtype not supported, device is not sm_100 */
  SV_ERR_CUDA = 3,        /* a CUDA runtime/driver call or a launch failed */
  SV_ERR_TIMEOUT = 4      /* a kernel's bounded wait expired (read through sv_device_status) */
} sv_status;

typedef enum { SV_BF16 = 0, SV_F32 = 1 } sv_dtype;

typedef enum {
  SV_OP_LINATTN_FWD = 0,
  SV_OP_BLOCK_STATE_UPDATE = 1,
  SV_OP_BLOCK_CAUSAL_ATTN = 2,
  SV_OP_CACHE_STEP = 3
} sv_op;

typedef struct CUstream_st* sv_stream_t; /* same type as cudaStream_t */

/* Bytes of workspace the call `op` needs for these sizes on the CURRENT device (the number of
 * streaming multiprocessors enters the size). block_len is read only for
 * SV_OP_BLOCK_CAUSAL_ATTN. Returns 0 for invalid sizes (see sv_last_error). */
size_t sv_workspace_bytes(sv_op op, int B, int H, int N, int D, int block_len, sv_dtype dt);

/* Zero the whole workspace (asynchronous on `stream`): the status word, the launch sequence words
 * and the flags between CTAs all start at zero. Call once after allocating. */
sv_status sv_workspace_init(void* ws, size_t ws_bytes, sv_stream_t stream);

/* Synchronise `stream`, read the workspace's status word and clear it. SV_OK if no kernel
 * raised it; SV_ERR_TIMEOUT if a bounded wait expired (the word is then in *code, if given).
 * Until it is cleared, a raised word makes every later call on this workspace give up its waits at
 * once (its output is then not written): a timeout is sticky, like a CUDA error. */
sv_status sv_device_status(void* ws, sv_stream_t stream, uint32_t* code);

/* Register a host word that the kernels also write when they raise the workspace's status word, so
 * that a caller learns of a device-side timeout without synchronising (for instance by checking the
 * word before each call, as the Python binding does). host_word must be page-locked host memory
 * that the device can write (cudaHostAlloc / cudaMallocHost; with unified addressing every such
 * allocation is mapped), 4-byte aligned, and must outlive the workspace's use; NULL removes the
 * registration. The caller clears host_word itself (sv_device_status clears only the device word).
 * Synchronises `stream`. Call after sv_workspace_init, which clears the registration. Returns
 * SV_ERR_INVALID_ARG for a bad workspace or a host_word the device cannot write. Not a step of the
 * method: failure reporting of this library. */
sv_status sv_workspace_set_mirror(void* ws, size_t ws_bytes, uint32_t* host_word, sv_stream_t stream);

/* Bidirectional full-sequence linear attention (the Linear DiT layer: every token attends to
 * every token of its (b, h) sequence; SANA-Video abstract, design (1) "Linear DiT"):
 *     o_i = phi(q_i) S / (phi(q_i) . z + eps),  S, z summed over all N tokens. */
sv_status sv_linattn_fwd(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int D,
                         sv_dtype dt, float eps, void* ws, size_t ws_bytes, sv_stream_t stream);

/* Add a block's state to the cache in place (talk, block KV cache passage: the state is updated
 * additively, the current block's contribution added to the previous cache):
 *     S += phi(K)^T V,  z += sum_j phi(k_j)  over the N tokens of k, v ([B, H, N, D]).
 * Unlike a plain cache update this call takes a workspace (sv_workspace_bytes with
 * SV_OP_BLOCK_STATE_UPDATE): the reduction is spread over every streaming multiprocessor, and their
 * partial states are combined there before S and z are written. */
sv_status sv_block_state_update(const void* k, const void* v, int B, int H, int N, int D, sv_dtype dt, float* S,
                                float* z, void* ws, size_t ws_bytes, sv_stream_t stream);

/* Block-causal prefill over a whole sequence cut into blocks of block_len tokens (the last block
 * may be shorter), as in the talk's block-causal walkthrough: block 1's state is cached, block 2's
 * contribution is added to that cache, and so on, so that every block sees the summed state of all
 * blocks before it; within its own block a token sees every token (the block is diffused as a
 * whole: talk, hybrid AR + diffusion passage). Token i of block c = floor(i / block_len) attends to
 * every token of blocks 0..c plus the incoming cache:
 *     P_c = S_in + sum_{c' <= c} S_c',  zP_c = z_in + sum_{c' <= c} z_c',
 *     o_i = phi(q_i) P_c / (phi(q_i) . zP_c + eps).
 * S_in/z_in (nullable: zero cache) is the cache before the sequence; S_out/z_out (nullable: not
 * written) receives the cache after the last block. S_out may equal S_in (in-place update).
 * block_len >= N is the bidirectional form. */
sv_status sv_block_causal_attn(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int D,
                               int block_len, sv_dtype dt, float eps, const float* S_in, const float* z_in,
                               float* S_out, float* z_out, void* ws, size_t ws_bytes, sv_stream_t stream);

/* One streaming step of the constant-memory cache (talk, block-causal walkthrough: the block's
 * output uses the cached state plus its own contribution; the new state is then cached): the
 * N tokens of q, k, v form one block, o = attention of the block over (block + cache). If
 * commit != 0 the cache then takes the block's state (S += phi(K)^T V, z += sum phi(k)); with
 * commit == 0 S and z are left untouched (e.g. the intermediate denoising steps of a block). */
sv_status sv_cache_step(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int D,
                        sv_dtype dt, float eps, float* S, float* z, int commit, void* ws, size_t ws_bytes,
                        sv_stream_t stream);

/* sv_cache_step without a workspace argument, for callers that cannot allocate device memory:
 * an operator called from a host framework that owns all memory, a real-time block loop that must
 * not call cudaMalloc (it synchronises the device), or code being recorded into a CUDA graph,
 * where allocation is not allowed while recording. The paper has no counterpart; this is a
 * deployment convenience of this library.
 * Scratch comes from one static device array of 16 MiB compiled into the library (held on every
 * device that loads the library until the process exits). Arguments and results are those of
 * sv_cache_step. A call that needs more scratch than 16 MiB (see sv_workspace_bytes with
 * SV_OP_CACHE_STEP: about 66 KB per (batch, head) pair plus 66 KB per streaming multiprocessor,
 * so the 720p streaming block [1, 20, 2760, 128] needs about 12 MB and B * H above ~100 does not
 * fit) is refused with SV_ERR_INVALID_ARG before any launch. All calls on a device share the
 * array, which keeps the previous call's contents: calls that may overlap on the GPU race. The
 * first call on a device looks up the array's device address and keeps it for the life of the
 * process; make it before any stream capture, and do not use this entry point across a
 * cudaDeviceReset. A device-side wait timeout raises the array's status word, which stays raised
 * (later calls then give up at once) until sv_cache_step_noalloc_status reads and clears it. */
sv_status sv_cache_step_noalloc(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int D,
                                sv_dtype dt, float eps, float* S, float* z, int commit, sv_stream_t stream);

/* sv_device_status for the static scratch of sv_cache_step_noalloc on the current device:
 * synchronises `stream`, reads the array's status word and clears it (SV_OK, or SV_ERR_TIMEOUT with
 * the word in *code if given). Allocates nothing. */
sv_status sv_cache_step_noalloc_status(sv_stream_t stream, uint32_t* code);

/* 3D rotary position embedding inside the linear attention (talk, passage on adapting the Linear
 * DiT to video: 3D RoPE for the linear attention; model-family page, architecture paragraph:
 * rotary position embeddings). The pages print no formula; this library reads it as follows.
 *  - The rotation acts on the feature-mapped q and k. It is applied to the numerator only; the
 *    normaliser keeps the unturned features, so that it stays positive:
 *        o_i = R_i phi(q_i) . P / (phi(q_i) . zP + eps),
 *        P = S_in + sum_j (R_j phi(k_j)) v_j^T,   zP = z_in + sum_j phi(k_j)   (visible j).
 *  - R_n turns the feature pairs (2p, 2p+1) by the angle pos * base^(-p'/P): the D/2 pairs are
 *    split into groups of pairs_t, pairs_h, pairs_w pairs (in that order) that take the token's
 *    frame, grid row and grid column as pos; p' is the pair's index in its group of P pairs.
 *  - Tokens are flattened frame-major on a grid of height x width tokens per frame: token n of a
 *    (batch, head) sequence sits at frame frame0 + n / (height*width), row (n / width) % height,
 *    column n % width.
 * The (cos, sin) table is built once per grid and feature split. */
typedef struct {
  const float* table; /* DEVICE table written by sv_rope3d_table with the fields below */
  int frames;         /* frame positions the table covers (0 .. frames-1) */
  int height, width;  /* tokens per frame: height rows x width columns */
  int D;              /* feature dimension of the table (even) */
  int pairs_t, pairs_h, pairs_w; /* pairs per group; 2 * (pairs_t + pairs_h + pairs_w) == D */
  int frame0;         /* frame of token 0 of q and k in the call; the call's last token must sit
                         inside the table: frame0 + (N-1) / (height*width) < frames */
} sv_rope3d;

/* Bytes of the table for `frames` frame positions, a height x width grid and feature dimension D:
 * (frames + height + width) * (D/2) * 8. 0 for arguments out of range (see sv_last_error). */
size_t sv_rope3d_table_bytes(int frames, int height, int width, int D);

/* Writes the (cos, sin) table into `table` (DEVICE, 16-byte aligned, table_bytes >=
 * sv_rope3d_table_bytes(...)): rows 0..frames-1 are frame positions, then `height` rows, then
 * `width` columns; each row holds D/2 fp32 (cos, sin) pairs, the angle of pair p' of the row's
 * group being pos * base^(-p'/P) computed in fp64 and rounded once; pairs of the other groups hold
 * (1, 0). base > 1 (10000 in RoFormer). One kernel on `stream`. */
sv_status sv_rope3d_table(float* table, size_t table_bytes, int frames, int height, int width, int D, int pairs_t,
                          int pairs_h, int pairs_w, float base, sv_stream_t stream);

/* sv_block_causal_attn with the 3D rotary embedding above (rope: HOST pointer to the descriptor,
 * read during the call). Arguments, outputs and the workspace (sv_workspace_bytes with
 * SV_OP_BLOCK_CAUSAL_ATTN) are those of sv_block_causal_attn. S_in / S_out hold the turned-key
 * state, z_in / z_out the unturned key sum, so one streaming step of the cache is this call with
 * block_len = N, S_in = S_out = S, z_in = z_out = z, and frame0 = the block's first frame;
 * block_len >= N is the bidirectional form. D must be even. The work always runs as the
 * three-kernel path (state, scan, output), also for one block per head. */
sv_status sv_block_causal_attn_rope(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int D,
                                    int block_len, sv_dtype dt, float eps, const float* S_in, const float* z_in,
                                    float* S_out, float* z_out, const sv_rope3d* rope, void* ws, size_t ws_bytes,
                                    sv_stream_t stream);

/* Block-causal temporal convolution of the causal Mix-FFN (talk, causal FFN with temporal conv
 * passage: a zero token is padded between two blocks so that block 1 cannot see block 2, and block
 * 2 takes block 1's last token as its first token so that it sees block 1; the padding and the
 * carried token are dropped after the convolution; the model-family page places a one-dimensional
 * temporal convolution inside the Mix-FFN). The pages give neither the width nor the weights; this
 * library reads the passage as a depthwise convolution along time with a centred kernel of width 3
 * (one padding token, one carried token), in cross-correlation order:
 *     y[t] = w[c][0] * x[t-1] + w[c][1] * x[t] + w[c][2] * x[t+1] * [blk(t+1) == blk(t)] + bias[c],
 * blk(t) = floor(t / frames_per_block), x[-1] = 0; the last block may be shorter.
 * x, y: DEVICE pointers to contiguous [B, T, S, C] tensors (T latent frames of S tokens, C channels,
 * C fastest), element type dt, 16-byte aligned; C a multiple of 8 (bf16) or 4 (fp32). y may equal x.
 * w: DEVICE fp32 [C][3]; bias: DEVICE fp32 [C] or NULL; both 16-byte aligned. Computed in fp32,
 * rounded once to dt. */
sv_status sv_temporal_conv(const void* x, void* y, int B, int T, int S, int C, int frames_per_block, const float* w,
                           const float* bias, sv_dtype dt, sv_stream_t stream);

/* One block of a stream through the same convolution: the T frames of x form one block; carry
 * (DEVICE [B, S, C] of dt, 16-byte aligned, zeros before the first block) is the previous block's
 * last frame, seen by frame 0 as its left neighbour; the block's last frame has the padding zero on
 * its right. If commit != 0, carry then receives x's last frame (in place). Memory kept between
 * blocks: carry only, whatever the number of blocks. Block by block this equals sv_temporal_conv of
 * the whole sequence (talk, causal FFN with temporal conv passage). */
sv_status sv_temporal_conv_step(const void* x, void* y, int B, int T, int S, int C, const float* w, const float* bias,
                                void* carry, int commit, sv_dtype dt, sv_stream_t stream);

/* The Q/K/V projection of a linear-attention layer with the feature map in its epilogue (SANA-Video
 * model-family page, 2.0 paragraph: hidden size 2560 = 20 heads x 128 features; the ReLU feature
 * map of the library's operation). The pages print no formula; this library's reading is a bias-free
 * linear map with one fused weight:
 *     [q | k | v] = x W_qkv^T,   q = ReLU(.),  k = ReLU(.),  v linear,
 * W_qkv [3*H*D, C] row-major bf16 (row f = output feature f: Q features 0..H*D-1, then K, then V;
 * head h owns features h*D .. h*D+D-1 of each). x: [B, N, C] bf16; q, k, v: [B, H, N, D] bf16 (the
 * layout the attention calls read; ReLU applied again there changes nothing). fp32 accumulation,
 * one bf16 rounding. All pointers are DEVICE pointers, 16-byte aligned. Supported: D = 64 or 128,
 * C a multiple of 64. ws: a workspace of at least 256 bytes (sv_workspace_init) whose status word
 * reports a device-side timeout (sv_device_status). */
sv_status sv_qkv_projection(const void* x, const void* w_qkv, void* q, void* k, void* v, int B, int N, int C, int H,
                            int D, void* ws, size_t ws_bytes, sv_stream_t stream);

/* The output projection after the attention (same page and reading): y = o_cat W_o^T with the
 * heads of o [B, H, N, D] concatenated feature-major (o_cat[b, n, h*D + d] = o[b, h, n, d], read in
 * place, no copy), W_o [C_out, H*D] row-major bf16, y [B, N, C_out] bf16. D = 64 or 128, C_out a
 * multiple of 64; ws as for sv_qkv_projection. */
sv_status sv_out_projection(const void* o, const void* w_o, void* y, int B, int N, int H, int D, int C_out, void* ws,
                            size_t ws_bytes, sv_stream_t stream);

/* Optional timing hook for benchmarks. With events != NULL (n == 4 cudaEvent_t handles owned by
 * the caller), the calling thread's following forward calls (sv_linattn_fwd, sv_block_causal_attn,
 * sv_cache_step) record events[0] before the state-reduction kernel, events[1] after it,
 * events[2] after the prefix scan and events[3] after the output kernel, on the call's stream.
 * When a call runs as a single launch (bf16, one block per head) events[1..3] all follow it.
 * Events between the kernels keep them from overlapping, so time with the hook removed.
 * events == NULL (n ignored) removes the hook. Costs one cudaEventRecord per mark. */
sv_status sv_profile_events(void* const* events, int n);

/* Message for the calling thread's most recent non-OK status ("" if none). */
const char* sv_last_error(void);

/* Failure-path self-test of the kernels' bounded waits; makes no GPU fault and leaves nothing in
 * flight. Launches one CTA whose waiters block, through the same bounded-wait routine the pipeline
 * kernels use, on an mbarrier phase that nothing completes. After the wait limit (about 2 s) the
 * first waiter raises the status word of `ws` to 0x80000000 | 0x7E00 | warp and every waiter
 * returns. Arguments: ws is a workspace (>= 256 bytes, 256-byte aligned, cleared by
 * sv_workspace_init); stream as for every call. Returns SV_OK once the kernel is launched
 * (SV_ERR_INVALID_ARG for a bad workspace, SV_ERR_CUDA if the launch fails); the expiry itself is
 * read afterwards with sv_device_status, which then returns SV_ERR_TIMEOUT and clears the word. */
sv_status sv_selftest_wait_timeout(void* ws, size_t ws_bytes, sv_stream_t stream);

/* Library version, major * 10000 + minor * 100 + patch. */
int sv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SVLINATTN_H */
