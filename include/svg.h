/*
 * svg.h -- C ABI of libsvg: spatial/temporal sparse 3D attention for video
 * diffusion transformers on NVIDIA B200 (sm_100a).
 *
 * The method (Sparse VideoGen) runs four steps right before each 3D attention
 * call:
 *   1. online profiling labels every head spatial or temporal
 *      (svg_profile_heads);
 *   2. the layout transformation moves temporal heads' Q/K/V from frame-major
 *      to token-major order (svg_permute / svg_permute_qkv);
 *   3. block-sparse attention over each head's block-banded pattern
 *      (svg_block_sparse_attn);
 *   4. the inverse layout transformation of the output (svg_unpermute).
 * svg_sparse_3d_attn runs all four.  svg_dense_attn is the unmasked reference.
 *
 * Sources, cited by page title and section:
 *   "Sparse Video-Gen" author rebuttal (paperhub.cn): Weakness 1 answer
 *     (token indexing x = i*F + j; Spatial Head mask |i1-i2| < a1; Temporal
 *     Head mask |j1-j2| < a2) and the later Weakness 1 answer on online
 *     profiling (per step and layer, right before attention; labels -1/+1).
 *   "Sparse VideoGen: Accelerating Video Diffusion Transformers with
 *     Spatial-Temporal Sparsity" (newx.sg): Abstract (online profiling,
 *     hardware-efficient layout transformation, custom kernels).
 *   SVG2 explainer (gist.science), 2.A "Semantic-Aware Permutation": a token
 *     permutation applied before attention and undone after it leaves the
 *     output unchanged.
 *
 * Conventions shared by every entry point
 *   Shapes.   B batch, H heads, N frames, F tokens per frame, L = N*F tokens,
 *             d head dim.  Token (i, j) (frame i, in-frame position j) sits at
 *             row x = i*F + j of the frame-major layout.
 *   Layout.   Every Q/K/V/O tensor argument of a call is contiguous, d
 *             fastest, in the element type of shape->dtype (bf16 or fp32),
 *             and ordered as shape->layout says: [B, H, L, d]
 *             (SVG_LAYOUT_BHLD, the default) or [B, L, H, d]
 *             (SVG_LAYOUT_BLHD, the heads of one token side by side, as a
 *             fused QKV projection writes them).  The arithmetic does not
 *             depend on the layout: every kernel gives bit-identical
 *             results on either (svg_sparse_3d_attn picks its plan per
 *             layout, see there).
 *             Token-major ("permuted") tensors have the same shape and
 *             layout with token (i, j) at row x' = j*N + i.  Workspaces are
 *             opaque.  svg_sparse_3d_attn_host takes [B, H, L, d] only.
 *   Labels.   int8 per (b, h), [B, H]: SVG_SPATIAL (0) or SVG_TEMPORAL (1),
 *             standing for the pages' -1 and +1.
 *   Memory.   The caller allocates and owns every buffer.  Pointers named
 *             *_dev or described as device memory are CUDA device pointers;
 *             tensor pointers must be 16-byte aligned.  No entry point
 *             allocates or frees memory or synchronises the stream.
 *   Streams.  `stream` is a cudaStream_t (NULL = legacy default stream).  All
 *             device work is enqueued asynchronously on it.
 *   Errors.   The return value reports argument errors (SVG_ERR_INVALID_ARG,
 *             SVG_ERR_UNSUPPORTED, SVG_ERR_WORKSPACE) before anything is
 *             enqueued, and launch errors (SVG_ERR_CUDA) after.  Errors that
 *             happen on the device (a bounded wait that ran out) are OR-ed
 *             into the optional device word `status_dev` as SVG_DEV_* bits;
 *             read it after the stream has synchronised.  With status_dev
 *             NULL they go to one word per device that every such call
 *             shares (and zeroes first), so calls that overlap on the GPU
 *             can clear each other's bits: pass a word of your own to rely
 *             on them.  svg_last_error() gives a message for the last
 *             failing call on this host thread.
 *   Support.  bf16: d in {64, 128}.  fp32 and tf32: d in {32, 64, 128}.  a1 >= 1,
 *             a2 >= 1 (a1 >= N or a2 >= F keep every pair of that kind).
 */
#ifndef SVG_H_
#define SVG_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SVG_API __attribute__((visibility("default")))
#else
#define SVG_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum svg_status {
  SVG_OK = 0,
  SVG_ERR_INVALID_ARG = 1, /* null pointer, bad size or band, misalignment */
  SVG_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. d = 96)      */
  SVG_ERR_CUDA = 3,        /* a CUDA call or launch failed                */
  SVG_ERR_TIMEOUT = 4,     /* reserved for host-side reporting of SVG_DEV_TIMEOUT */
  SVG_ERR_WORKSPACE = 5    /* workspace smaller than the size query says   */
} svg_status;

/* Element type of the Q/K/V/O tensors and the arithmetic of attention:
 * SVG_BF16  bf16 tensors, tcgen05 kind::f16 products, fp32 softmax and
 *           accumulation, bf16 output;
 * SVG_FP32  fp32 tensors, fp32 arithmetic on the CUDA cores (the exact path);
 * SVG_TF32  fp32 tensors, attention products on the tcgen05 tensor cores in
 *           tf32 (kind::tf32: 10-bit mantissas), fp32 softmax, accumulation
 *           and output; profiling, permutation and labels as SVG_FP32. */
typedef enum svg_dtype { SVG_BF16 = 0, SVG_FP32 = 1, SVG_TF32 = 2 } svg_dtype;

#define SVG_SPATIAL 0
#define SVG_TEMPORAL 1

/* Bits of the device status word. */
#define SVG_DEV_TIMEOUT 0x1u  /* a pipeline wait exceeded its bound; outputs invalid */
#define SVG_DEV_RANGE 0x2u    /* profiling: in-band weights underflowed (see svg_profile_heads);
                                 semantic attention: a cluster id out of range */
#define SVG_DEV_BOUNDS 0x4u   /* debug build only: a kernel index outside its buffer (the access was
                                 skipped; see svg_debug_checks) */

/* Order of the Q/K/V/O tensors of a call (svg_shape.layout). */
#define SVG_LAYOUT_BHLD 0 /* [B, H, L, d]: each head's L rows are contiguous */
#define SVG_LAYOUT_BLHD 1 /* [B, L, H, d]: row x of head h is H*d elements after row x - 1 */

typedef struct svg_shape {
  int32_t B, H, N, F, d;
  int32_t dtype;  /* svg_dtype */
  float scale;    /* softmax scale on q.k; 0 selects 1/sqrt(d) */
  int32_t layout; /* SVG_LAYOUT_*; a zero-initialised shape is [B, H, L, d] */
} svg_shape;

/* ABI version of this header (bumped on any signature or struct change). */
#define SVG_ABI_VERSION 2
SVG_API int32_t svg_abi_version(void);

/* Static text for a status code; never NULL. */
SVG_API const char* svg_status_string(int32_t status);

/* Message for the last non-OK status returned on the calling host thread. */
SVG_API const char* svg_last_error(void);

/*
 * svg_debug_checks -- 1 if this library was built with range checks
 * (libsvg_debug.so, compiled with SVG_DEBUG_BOUNDS=1), 0 otherwise.  In the
 * checked build every global-memory index the tensor-core kernels compute
 * (output rows, sampled rows, workspace slots, cluster ids and offsets, TMA
 * tile coordinates) is compared with its buffer first; an index outside it
 * sets SVG_DEV_BOUNDS in the status word and the store is skipped, so a
 * wrong index is reported instead of faulting or trapping.  Shared-memory and
 * tensor-memory offsets are fixed per kernel and checked at compile time.
 * The checked build is slower and meant for tests.
 */
SVG_API int32_t svg_debug_checks(void);

/*
 * svg_attn_tile -- query/key tile sizes (rows) of the attention kernel for a
 * given dtype and head dim, i.e. the Bq x Bk tiling its block list refers to.
 * Host only.
 */
SVG_API svg_status svg_attn_tile(int32_t dtype, int32_t d, int32_t* Bq, int32_t* Bk);

/*
 * svg_block_list -- the block schedule of a block-banded mask, host only.
 *
 * Mask: keep (x, y) iff |floor(x/G) - floor(y/G)| < a over L tokens.  With
 * G = F, a = a1 this is the spatial mask ("Sparse Video-Gen", Spatial Head:
 * block-banded with the main and +-(a1-1) neighbouring block diagonals); with
 * G = N, a = a2 it is the temporal mask after the token-major layout
 * transformation.  For each query tile qb (rows [qb*Bq, min(L,(qb+1)*Bq))),
 * writes the key-tile ranges [kb_lo[qb], kb_hi[qb]) of tiles with any kept
 * element and [full_lo[qb], full_hi[qb]) of tiles with every element kept
 * (an empty range has lo == hi).  These are the tiles the attention kernel
 * visits and the ones it visits without an elementwise mask.
 * Arrays: host memory, ceil(L/Bq) int32 each, owned by the caller.
 * Errors: SVG_ERR_INVALID_ARG if L, G, a, Bq or Bk < 1 or a pointer is NULL.
 */
SVG_API svg_status svg_block_list(int32_t L, int32_t G, int32_t a, int32_t Bq, int32_t Bk,
                          int32_t* kb_lo, int32_t* kb_hi, int32_t* full_lo, int32_t* full_hi);

/*
 * svg_profile_workspace_size -- bytes of device workspace svg_profile_heads
 * needs for this shape and sample count (0 on invalid arguments): the
 * per-chunk partial results, the per-row sums and the call's own device
 * status word.
 */
SVG_API size_t svg_profile_workspace_size(const svg_shape* shape, int32_t S);

/*
 * svg_workspace_size -- bytes of device workspace the step-by-step call needs
 * (svg_profile_heads -> svg_permute_qkv -> svg_block_sparse_attn ->
 * svg_unpermute) besides the caller's q, k, v and o, for any sample count
 * S <= 128 and at most n_temporal_heads_max temporal heads.  Layout, each part
 * starting on a 256-byte boundary: [profiling workspace | qp | kp | vp | op].
 * The four token-major tensors are present only when n_temporal_heads_max > 0,
 * each the size of q: a temporal head's token-major copy sits at its own head
 * index of a [B,H,L,d] tensor, so they do not shrink with fewer temporal heads.
 * The whole call sizes its own workspace (svg_sparse_3d_attn_workspace_size).
 * Returns 0 on invalid arguments (invalid shape, n_temporal_heads_max < 0 or
 * > B*H).
 */
SVG_API size_t svg_workspace_size(const svg_shape* shape, int32_t n_temporal_heads_max);

/*
 * svg_profile_heads -- online profiling ("Sparse Video-Gen", Weakness 1
 * answer on online profiling; "Sparse VideoGen ...", Abstract).
 *
 * For every head (b, h) and every sampled query row x = rows[s], computes
 * the exact attention output of that row with no mask (O_dense), under the
 * spatial mask |i_x - i_y| < a1 (O_s) and under the temporal mask
 * |j_x - j_y| < a2 (O_t), in fp32 from the given inputs, then
 *   mse[b,h,0] = mean over S*d of (O_s - O_dense)^2,
 *   mse[b,h,1] = mean over S*d of (O_t - O_dense)^2,
 *   label[b,h] = SVG_TEMPORAL if mse[b,h,1] < mse[b,h,0] else SVG_SPATIAL.
 * The reduction order is fixed, so repeated calls give identical bits.
 * The three softmaxes of a row share one reference (the row's running max
 * over the keys of a key chunk, a contiguous range of keys the kernel takes
 * as one unit of work), so every key needs one exponential.  If, within one
 * chunk, a row's in-band logits all lie more than about 126 / (scale *
 * log2(e)) below its largest logit of that chunk (about 990 raw units for
 * d = 128), their weights underflow.  That
 * case, like a device-side wait that ran out, is reported rather than
 * returned: every label is set to -1 and every MSE to NaN.  The call keeps
 * its status word inside the workspace (zeroed at the start of the call), so
 * calls with separate workspaces never see each other's failures; the whole
 * calls (svg_sparse_3d_attn, svg_sparse_3d_attn_host) also OR the failure
 * bits (SVG_DEV_RANGE, SVG_DEV_TIMEOUT) into their status_dev.  The
 * attention entry points run a head whose label is not SVG_TEMPORAL (-1
 * included) with the spatial band.
 *
 * q, k, v   device, [B,H,L,d] frame-major, dtype of shape.
 * rows      device, int32 [S], each in [0, L) (duplicates allowed), shared by
 *           every head.  1 <= S <= 128.
 * mse       device, float [B,H,2] (written).
 * label     device, int8 [B,H] (written).
 * workspace device, >= svg_profile_workspace_size(shape, S) bytes, 256-byte
 *           aligned; contents on entry do not matter.
 * Errors: SVG_ERR_INVALID_ARG (null pointer, S out of range, a1/a2 < 1),
 *         SVG_ERR_UNSUPPORTED (dtype/d), SVG_ERR_WORKSPACE, SVG_ERR_CUDA.
 */
SVG_API svg_status svg_profile_heads(const svg_shape* shape, const void* q, const void* k, const void* v,
                             int32_t a1, int32_t a2, const int32_t* rows, int32_t S, float* mse,
                             int8_t* label, void* workspace, size_t workspace_bytes, void* stream);

/*
 * svg_profile_heads_noalloc -- svg_profile_heads for callers that cannot
 * allocate device memory.  The pages describe nothing like it; it exists for
 * integration only.
 *
 * Who needs it: code that is handed only its input and output tensors and
 * has no allocator of its own (a plugin inside a host framework that owns
 * all device memory), and loops that must never call cudaMalloc, because
 * that call can synchronise the whole device at an unpredictable moment.
 * Instead of a caller workspace, this variant uses a fixed scratch array of
 * SVG_PROFILE_NOALLOC_SCRATCH_BYTES that lives in the library's device image.
 * Every GPU on which the library is used holds that array until the process
 * exits.  It computes the same quantities as svg_profile_heads.  When the
 * default key split would not fit the array, it splits the keys into fewer
 * chunks, so results can differ from svg_profile_heads in the last bits.
 *
 * Set-up: the first call on a device looks up the array's device address
 * (which also loads the library's kernels on that device) and remembers it.
 * Make that first call before any stream capture on that device.  The
 * remembered address belongs to the device's current CUDA context: after
 * cudaDeviceReset the call must not be used again in the process.
 * Failures on the device are recorded in a status word inside the array.
 * Sharing: every call on a device uses the same array, which keeps the last
 * call's contents.  Nothing in it needs to start at zero, because each call
 * writes every byte it later reads.  Calls whose kernels overlap on the GPU,
 * for example on two streams, race on the array: serialise them.
 * Limits: shapes whose partial results cannot fit the array even with one
 * key chunk return SVG_ERR_WORKSPACE before anything is enqueued.  The call allocates and
 * frees nothing.  Arguments are otherwise as for svg_profile_heads.
 */
#define SVG_PROFILE_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
SVG_API svg_status svg_profile_heads_noalloc(const svg_shape* shape, const void* q, const void* k,
                                             const void* v, int32_t a1, int32_t a2, const int32_t* rows,
                                             int32_t S, float* mse, int8_t* label, void* stream);

/*
 * svg_permute -- the layout transformation ("Sparse VideoGen ...", Abstract;
 * SVG2 explainer 2.A) of one tensor: for every head with label[b,h] ==
 * SVG_TEMPORAL, xp[b,h, j*N+i, :] = x[b,h, i*F+j, :].  Rows of spatial heads
 * in xp are not written.  label == NULL permutes every head.
 * x, xp: device [B,H,L,d], distinct, 16-byte aligned.  label: device or NULL.
 */
SVG_API svg_status svg_permute(const svg_shape* shape, const void* x, void* xp, const int8_t* label,
                       void* stream);

/* svg_permute_qkv -- svg_permute of q, k and v in one launch. */
SVG_API svg_status svg_permute_qkv(const svg_shape* shape, const void* q, const void* k, const void* v,
                           void* qp, void* kp, void* vp, const int8_t* label, void* stream);

/*
 * svg_unpermute -- inverse layout transformation: for every head with
 * label[b,h] == SVG_TEMPORAL, x[b,h, i*F+j, :] = xp[b,h, j*N+i, :].  Rows of
 * spatial heads in x are not written.  label == NULL unpermutes every head.
 */
SVG_API svg_status svg_unpermute(const svg_shape* shape, const void* xp, void* x, const int8_t* label,
                         void* stream);

/*
 * svg_block_sparse_attn -- block-sparse attention over each head's banded
 * pattern (the "customized kernel" of "Sparse VideoGen ...", Abstract; masks
 * from "Sparse Video-Gen", Spatial Head / Temporal Head).
 *
 *   spatial head:  O = softmax(scale*QK^T + M)V on q,k,v -> o, with M = 0 iff
 *                  |floor(x/F) - floor(y/F)| < a1 (frame-major rows);
 *   temporal head: the same on qp,kp,vp -> op with G = N, a = a2, i.e.
 *                  |floor(x'/N) - floor(y'/N)| < a2 on token-major rows, which
 *                  is the temporal mask |j1-j2| < a2 after the layout
 *                  transformation.
 * All heads run in one launch; the key range of each query tile is computed
 * on the fly from (G, a); no mask tensor is read.  Rows of temporal heads in
 * o and of spatial heads in op are not written.  A label other than
 * SVG_TEMPORAL (for instance the -1 of a failed profiling call) is treated
 * as SVG_SPATIAL, as by the permute and unpermute calls, which move only
 * SVG_TEMPORAL heads.
 *
 * q,k,v,o      device [B,H,L,d] frame-major.
 * qp,kp,vp,op  device [B,H,L,d] token-major (temporal heads' slices are used);
 *              may be NULL when no head is temporal.
 * label        device int8 [B,H].
 * status_dev   device int32 or NULL (SVG_DEV_* bits OR-ed in).
 */
SVG_API svg_status svg_block_sparse_attn(const svg_shape* shape, const void* q, const void* k,
                                 const void* v, const void* qp, const void* kp, const void* vp,
                                 void* o, void* op, const int8_t* label, int32_t a1, int32_t a2,
                                 int32_t* status_dev, void* stream);

/*
 * svg_banded_attn -- the same kernel with one band for every head:
 * keep (x, y) iff |floor(x/G) - floor(y/G)| < a, on q,k,v -> o as given
 * (no label, no permutation).  G >= L or a large gives dense attention.
 */
SVG_API svg_status svg_banded_attn(const svg_shape* shape, const void* q, const void* k, const void* v,
                           void* o, int32_t G, int32_t a, int32_t* status_dev, void* stream);

/*
 * svg_dense_attn -- unmasked attention softmax(scale*QK^T)V of every head,
 * the reference the sparse call is compared with.  Same kernel, one band
 * covering all L tokens.
 */
SVG_API svg_status svg_dense_attn(const svg_shape* shape, const void* q, const void* k, const void* v,
                          void* o, int32_t* status_dev, void* stream);

/*
 * svg_sparse_3d_attn_workspace_size -- bytes of device workspace the whole
 * call needs for temporal band a2 and S sampled rows: the profiling
 * workspace, plus token-major copies of q, k, v and o unless the call folds
 * the layout transformation into attention (see svg_sparse_3d_attn).  0 on
 * invalid arguments.
 */
SVG_API size_t svg_sparse_3d_attn_workspace_size(const svg_shape* shape, int32_t a2, int32_t S);

/*
 * svg_sparse_3d_attn_plan -- the layout choice svg_sparse_3d_attn makes, on
 * the host: separate_tiles / fused_tiles = 128-key tiles one temporal head
 * takes over all its query rows with token-major copies / with the fused
 * frame-group layout; *fused = 1 if the call folds the layout transformation
 * into attention.  Host pointers.
 */
SVG_API svg_status svg_sparse_3d_attn_plan(const svg_shape* shape, int32_t a2, int64_t* separate_tiles,
                                           int64_t* fused_tiles, int32_t* fused);

/*
 * svg_sparse_3d_attn -- one whole sparse 3D-attention call, enqueued on
 * `stream` with no host synchronisation: profile -> block-sparse attention
 * with the layout transformation fused in (svg_block_sparse_attn_fused), or
 * profile -> permute temporal heads -> block-sparse attention -> unpermute.
 * The fused form is used for bf16 [B, H, L, d] tensors when its frame-group
 * tiling costs at most 3 % more attention work than the token-major copies
 * (about what the two permutation passes cost), counted on the host from N,
 * F and a2; fp32 and [B, L, H, d] tensors always permute (in [B, L, H, d]
 * the fused boxes span the whole tensor and measured slower than the
 * copies, which the workspace holds as [B, H, L, d]).  Results are
 * bit-identical across layouts for the same plan; the two plans differ in
 * the order keys are summed (rounding only).  Outputs o (frame-major [B,H,L,d]) plus the profiling
 * results mse [B,H,2] and label [B,H] (device).  If profiling fails on the
 * device (see svg_profile_heads), its SVG_DEV_* bits are OR-ed into
 * status_dev and every head, labelled -1, gets the spatial attention; both
 * layouts give that same output.  Arguments as in the calls above.
 */
SVG_API svg_status svg_sparse_3d_attn(const svg_shape* shape, const void* q, const void* k, const void* v,
                              void* o, int32_t a1, int32_t a2, const int32_t* rows, int32_t S,
                              float* mse, int8_t* label, void* workspace, size_t workspace_bytes,
                              int32_t* status_dev, void* stream);

/*
 * svg_sparse_3d_attn_host_workspace_size -- device workspace of
 * svg_sparse_3d_attn_host for a chunk of `heads_per_chunk` heads (0 on bad
 * arguments): two slots, each with a chunk's q, k, v, o, their token-major
 * copies when svg_sparse_3d_attn would make them, and the chunk's profiling
 * workspace.
 */
SVG_API size_t svg_sparse_3d_attn_host_workspace_size(const svg_shape* shape, int32_t a2, int32_t S,
                                                      int32_t heads_per_chunk);

/*
 * svg_sparse_3d_attn_host -- svg_sparse_3d_attn on HOST buffers.
 *
 * q_host, k_host, v_host, o_host: [B,H,L,d] in host memory, page-locked for the
 * copies to overlap (pageable memory works, but the copies then serialise);
 * shape->layout must be SVG_LAYOUT_BHLD (a chunk of heads is then one
 * contiguous copy), else SVG_ERR_UNSUPPORTED;
 * rows_host [S], mse_host [B,H,2], label_host [B,H] in host memory.  Heads
 * are independent, so the call is cut into chunks of heads_per_chunk heads.
 * The host-to-device copies of one chunk, the kernels of another and the
 * device-to-host copies of a third overlap on two internal streams plus the
 * caller's stream.  The results are bit-identical to svg_sparse_3d_attn.
 * The call is asynchronous: `stream` resumes after the last copy-out, so
 * synchronise it before reading the host outputs.  The internal streams
 * and events are shared per device, so calls on one device from several
 * host threads take a per-device lock while they enqueue (their work then
 * runs in that order on the shared copy streams).
 */
SVG_API svg_status svg_sparse_3d_attn_host(const svg_shape* shape, const void* q_host, const void* k_host,
                                           const void* v_host, void* o_host, int32_t a1, int32_t a2,
                                           const int32_t* rows_host, int32_t S, float* mse_host,
                                           int8_t* label_host, int32_t heads_per_chunk, void* workspace,
                                           size_t workspace_bytes, int32_t* status_dev, void* stream);

/*
 * Head sharding across GPUs.  Every head's profiling, layout transformation
 * and attention touch no other head, so one call splits over `world` ranks
 * (one process per GPU) by head with no exchange on the data path.  Heads are
 * numbered over (b, h) as g = b * H + h; rank r takes the contiguous block
 * [first, first + count) with count = n / world or n / world + 1 (the first
 * n % world ranks take one more), so the blocks cover every head exactly once.
 *
 * svg_head_shard -- that block for n_heads heads (host only; 0 <= rank <
 * world; count may be 0 when world > n_heads).
 */
SVG_API svg_status svg_head_shard(int32_t n_heads, int32_t rank, int32_t world, int32_t* first, int32_t* count);

/*
 * svg_sparse_3d_attn_shard_workspace_size / svg_sparse_3d_attn_shard --
 * svg_sparse_3d_attn on this rank's block of heads only.  q, k, v, o, mse and
 * label are the FULL tensors on this rank's device, in shape->layout as for
 * svg_sparse_3d_attn; heads are numbered over (b, h), so in [B, L, H, d] a
 * block can end in one batch entry and go on in the next.  Only the block's
 * heads are read and written, so a caller that wants the whole output
 * gathers the blocks from the other ranks afterwards (one all-gather over
 * NVLink), and a caller that keeps heads sharded never does.  The workspace
 * is sized for the block.  With no heads on this rank the call does nothing
 * and returns SVG_OK.
 */
SVG_API size_t svg_sparse_3d_attn_shard_workspace_size(const svg_shape* shape, int32_t rank, int32_t world,
                                                       int32_t a2, int32_t S);
SVG_API svg_status svg_sparse_3d_attn_shard(const svg_shape* shape, int32_t rank, int32_t world, const void* q,
                                            const void* k, const void* v, void* o, int32_t a1, int32_t a2,
                                            const int32_t* rows, int32_t S, float* mse, int8_t* label,
                                            void* workspace, size_t workspace_bytes, int32_t* status_dev,
                                            void* stream);

/*
 * Mixed sparse patterns ("Sparse-vDiT" review, pith.science, "What carries
 * the argument": every head takes one of five modes -- full attention, skip,
 * diagonal, multi-diagonal, vertical stripe -- and heads that share a mode
 * are fused into one operation; the multi-diagonal pattern is handled by a
 * token rearrangement that turns it into a diagonal one).  Per-head modes,
 * as int8 values in a device array [B, H]:
 *   SVG_MODE_FULL       every key
 *   SVG_MODE_SKIP       no key: the head's output is zero
 *   SVG_MODE_DIAGONAL   |x - y| <= window (a band of width 2*window + 1)
 *   SVG_MODE_MULTIDIAG  |j_x - j_y| <= md_half: the same in-frame position
 *                       (+-md_half) in every frame, i.e. diagonals of stride F;
 *                       run on token-major copies, where it is block-banded
 *                       with G = N and a = md_half + 1
 *   SVG_MODE_STRIPE     y < stripe (the first `stripe` keys)
 */
#define SVG_MODE_FULL 0
#define SVG_MODE_SKIP 1
#define SVG_MODE_DIAGONAL 2
#define SVG_MODE_MULTIDIAG 3
#define SVG_MODE_STRIPE 4

/*
 * svg_mixed_attn -- attention of every head under its own mode, all heads in
 * one launch (bf16 only).  Multi-diagonal heads read qp,kp,vp (token-major)
 * and write op; every other head reads q,k,v and writes o (skipped heads
 * write zeros to o).  window, md_half >= 0; stripe >= 1.  Other arguments as
 * for svg_block_sparse_attn.
 */
SVG_API svg_status svg_mixed_attn(const svg_shape* shape, const void* q, const void* k, const void* v,
                                  const void* qp, const void* kp, const void* vp, void* o, void* op,
                                  const int8_t* mode, int32_t window, int32_t md_half, int32_t stripe,
                                  int32_t* status_dev, void* stream);

/* svg_mixed_3d_attn_workspace_size -- workspace of svg_mixed_3d_attn (bytes; 0 on bad arguments). */
SVG_API size_t svg_mixed_3d_attn_workspace_size(const svg_shape* shape);

/*
 * svg_mixed_3d_attn -- one mixed-pattern attention call: permute the
 * multi-diagonal heads' q, k, v to token-major order, run svg_mixed_attn,
 * and permute their output back into o (frame-major [B,H,L,d]).
 */
SVG_API svg_status svg_mixed_3d_attn(const svg_shape* shape, const void* q, const void* k, const void* v, void* o,
                                     const int8_t* mode, int32_t window, int32_t md_half, int32_t stripe,
                                     void* workspace, size_t workspace_bytes, int32_t* status_dev,
                                     void* stream);

/*
 * svg_mode_search_workspace_size -- workspace of svg_mode_search (bytes; 0 on
 * bad arguments).
 */
SVG_API size_t svg_mode_search_workspace_size(const svg_shape* shape, int32_t S);

/*
 * svg_mode_search -- per-head mode selection of the mixed sparse patterns
 * ("Sparse-vDiT" review, "What carries the argument" and the referee report
 * on Sec. 4.2, Eq. (2)).  For each head and each sparse mode i in (skip,
 * diagonal, multi-diagonal, vertical stripe):
 *   L_i = MSE(O_i - O_dense) + lambda * (1 - S_i),
 * where the MSE is over the sampled rows and d (as in svg_profile_heads), O_i
 * is the attention under mode i (zero for skip), and S_i is the share of
 * (query, key) pairs the mode skips (1 for skip).  The head gets the mode with
 * the smallest L_i, or SVG_MODE_FULL if every L_i exceeds epsilon.
 * loss: device float [B,H,4] in the order skip, diagonal, multi-diagonal,
 * stripe.  mode: device int8 [B,H] (SVG_MODE_*; -1 if a device-side wait ran
 * out or in-band weights underflowed, with the losses set to NaN).
 * bf16 only; other arguments as for svg_profile_heads and svg_mixed_attn.
 */
SVG_API svg_status svg_mode_search(const svg_shape* shape, const void* q, const void* k, const void* v,
                                   const int32_t* rows, int32_t S, int32_t window, int32_t md_half,
                                   int32_t stripe, float lambda, float epsilon, float* loss, int8_t* mode,
                                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * svg_block_sparse_attn_fused -- svg_block_sparse_attn with the layout
 * transformation folded into the attention kernel.  The token-major order of
 * temporal heads ("Sparse VideoGen", Abstract: the hardware-efficient tensor
 * layout transformation; Sparse VideoGen2 review, 2.A on permuting before
 * attention and undoing it after) is applied while loading.  The N frames
 * are split into groups of power-of-two size s; one 128-row tile is s frames
 * x 128/s consecutive positions, loaded as one box of a 4D view of the
 * frame-major q/k/v, and already in token-major order.  Keys are visited
 * group by group (the temporal mask depends on the position only), and each
 * output row is written to its frame-major position in o.  No permuted
 * copies exist; o is frame-major for every head.  The key order differs from
 * the unfused path, so results agree with it to rounding, not bit for bit.
 * q, k, v, o: device bf16 [B,H,N*F,d] (d = 64 or 128); other arguments as
 * for svg_block_sparse_attn.  SVG_ERR_UNSUPPORTED for fp32.
 */
SVG_API svg_status svg_block_sparse_attn_fused(const svg_shape* shape, const void* q, const void* k, const void* v,
                                               void* o, const int8_t* label, int32_t a1, int32_t a2,
                                               int32_t* status_dev, void* stream);

/*
 * svg_mixed_attn_fused -- svg_mixed_attn with the multi-diagonal heads'
 * token-major layout folded in the same way (no permuted copies, o
 * frame-major for every head).  The whole mixed-pattern call in one launch.
 */
SVG_API svg_status svg_mixed_attn_fused(const svg_shape* shape, const void* q, const void* k, const void* v, void* o,
                                        const int8_t* mode, int32_t window, int32_t md_half, int32_t stripe,
                                        int32_t* status_dev, void* stream);

/*
 * svg_semantic_attn_workspace_size -- workspace of svg_semantic_attn (bytes;
 * 0 on bad arguments, fp32, or cluster counts outside [1, 1024]).
 */
SVG_API size_t svg_semantic_attn_workspace_size(const svg_shape* shape, int32_t Cq, int32_t Ck);

/*
 * svg_semantic_attn -- SVG2-style sparse attention given each token's
 * cluster (SVG2 explainer, 2.A "Semantic-Aware Permutation", 2.B
 * "Centroid-Based Top-p Selection", 2.C "Customized Attention Kernel"):
 *   1. rows of Q are ordered by query cluster and rows of K, V by key
 *      cluster (stable: clusters in index order, rows in original order);
 *   2. each cluster's centroid is the mean of its rows;
 *   3. for query cluster c_q, key cluster c_k gets the mass
 *      n_k exp(scale mu_q . mu_k) (normalised over c_k; empty clusters 0);
 *      clusters are taken by mass, descending (ties: lower index), until the
 *      kept mass reaches p;
 *   4. each query row attends to every key of the key clusters its cluster
 *      keeps (one launch of the tcgen05 attention kernel over runs of kept
 *      clusters), and its output lands at its original row of o.
 * q, k, v, o: device bf16 [B,H,N*F,d], d = 64 or 128 (o frame-major like q).
 * assign_q, assign_k: device int32 [B,H,L] cluster ids in [0, Cq) / [0, Ck)
 *   (an id out of range sets SVG_DEV_RANGE in *status_dev and is read as 0).
 * p in (0, 1].  selected: device uint32 [B,H,Cq,ceil(Ck/32)], written: bit c_k
 * of word c_k/32 is set iff query cluster c_q keeps key cluster c_k.
 * workspace: svg_semantic_attn_workspace_size bytes, 256-byte aligned.
 * Deterministic: repeated calls return the same bits.
 */
SVG_API svg_status svg_semantic_attn(const svg_shape* shape, const void* q, const void* k, const void* v, void* o,
                                     const int32_t* assign_q, const int32_t* assign_k, int32_t Cq, int32_t Ck,
                                     float p, uint32_t* selected, void* workspace, size_t workspace_bytes,
                                     int32_t* status_dev, void* stream);

/*
 * svg_kmeans_workspace_size / svg_kmeans -- k-means of every head's rows of x
 * (SVG2 explainer, 2.A: Q and K are clustered independently by k-means).
 * Lloyd's algorithm, `iters` rounds from the rows floor(c L / C): each row
 * goes to the nearest centroid (squared Euclidean distance, the centroid
 * rounded to bf16 for the product, ties to the lower index; tcgen05 GEMM with
 * the argmin in its epilogue), then each centroid becomes the mean of its
 * rows (fp32, summed in the rows' original order; an empty cluster keeps its
 * centroid).  Outputs: assign device int32 [B,H,L] (the last round's) and
 * centroids device float [B,H,C,d] (the means of that assignment).
 * x: device bf16 [B,H,N*F,d], d = 64 or 128; 1 <= C <= min(512, L).
 * Deterministic.  The size query returns 0 on bad arguments.
 */
SVG_API size_t svg_kmeans_workspace_size(const svg_shape* shape, int32_t C);
SVG_API svg_status svg_kmeans(const svg_shape* shape, const void* x, int32_t C, int32_t iters, int32_t* assign,
                              float* centroids, void* workspace, size_t workspace_bytes, int32_t* status_dev,
                              void* stream);

/*
 * svg_semantic_3d_attn_workspace_size / svg_semantic_3d_attn -- the whole
 * SVG2-style call: svg_kmeans of Q into Cq clusters and of K into Ck clusters
 * (`iters` rounds each), then svg_semantic_attn with keep threshold p.
 * Outputs o, assign_q / assign_k (device int32 [B,H,L]) and selected (as in
 * svg_semantic_attn).  Cluster counts 1..512.
 */
SVG_API size_t svg_semantic_3d_attn_workspace_size(const svg_shape* shape, int32_t Cq, int32_t Ck);
SVG_API svg_status svg_semantic_3d_attn(const svg_shape* shape, const void* q, const void* k, const void* v, void* o,
                                        int32_t Cq, int32_t Ck, int32_t iters, float p, int32_t* assign_q,
                                        int32_t* assign_k, uint32_t* selected, void* workspace,
                                        size_t workspace_bytes, int32_t* status_dev, void* stream);

/*
 * svg_selftest_wait_bound -- failure-detection self-test (test hook).
 *
 * Runs the bf16 attention kernel (one band covering all keys) with its
 * producer's loads withheld, so nothing ever arrives on the barriers its
 * consumers wait for.  Every wait must give up after wait_ns.  The kernel
 * then sets SVG_DEV_TIMEOUT in *status_dev, frees its tensor memory and
 * exits; CTAs that start later see the bit and skip their work.  The CUDA
 * context stays usable.  o is left unspecified.  The call itself returns
 * SVG_OK once the launch is enqueued.
 * wait_ns in [1e6, 1e10]; status_dev is required and must be zero on entry.
 */
SVG_API svg_status svg_selftest_wait_bound(const svg_shape* shape, const void* q, const void* k,
                                           const void* v, void* o, uint64_t wait_ns,
                                           int32_t* status_dev, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SVG_H_ */
