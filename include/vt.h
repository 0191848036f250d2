/*
 * vt.h — C ABI of libvt, a B200 (sm_100a) implementation of the forward pass of a
 * CLIP-style ViT vision tower with a 2x2-merge projector, with variable-resolution
 * batches, video clips, GPU preprocessing of decoded images and the backward pass to the
 * pixels.
 *
 * The model is the one described by the "MiniMax-M3 Vision" model card (Architecture
 * table): patch 14, Conv3d patch embedding with temporal patch 2, 32 pre-LN layers of
 * hidden 1280, 16 heads, MLP 5120 with GELU, 3D RoPE; a 2x2 spatial merge; the
 * projector Linear(1280,6144), GELU, Linear(6144,6144), flatten four 6144-wide tokens
 * to 24576, Linear(24576,6144), GELU, Linear(6144,6144).
 *
 * Conventions shared by every entry point
 *  - Pointers named "device" are CUDA device addresses on the current device; "host"
 *    pointers are ordinary CPU memory.  bf16 tensors are passed as void* holding IEEE
 *    bfloat16 values (1 sign, 8 exponent, 7 mantissa bits), row-major, dense.
 *  - All device pointers must be 16-byte aligned.
 *  - Ownership: the library never frees caller memory.  Weights passed to
 *    vt_load_weights are borrowed and must outlive the handle.  Workspaces are owned by
 *    the caller.  The library's only device memory is the handle's fused QKV weight
 *    pack (when q, k, v are loaded separately), its RoPE cos/sin tables, the transposed
 *    weights of vt_enable_backward, and the fixed scratch of vt_attention_static.
 *  - Every compute call is asynchronous on the given stream (a cudaStream_t passed as
 *    void*, NULL = legacy default stream), allocates nothing and does not synchronise,
 *    except vt_load_weights, vt_enable_backward, vt_destroy, vt_check and
 *    vt_forward_host as documented.
 *  - Errors: every call returns a vt_status.  Argument errors are detected on the host
 *    before anything is launched.  vt_last_error() returns a message for the last
 *    failure of the calling thread.  No C++ exception crosses this interface.
 *  - Kernels bound every internal wait (1 s); a wait that runs out records a device
 *    error that vt_check() reports as VT_ERR_TIMEOUT.
 *  - Tracing: with the environment variable VT_LOG set (not empty, not "0") when the
 *    library loads, every kernel launch is written to stderr as it is issued: its
 *    class, algorithmic FLOPs and bytes, and stream.  vt_profile_* time the launches.
 *  - Devices: one process drives one GPU (the library's deployment model; several GPUs
 *    run one process each).  Each kernel's shared-memory attribute is set once per
 *    process, on the device current at its first launch, so a process that switches
 *    the current device between calls is not supported.
 *  - Token order: activations of one image are t*h*w tokens.  Raster order puts token
 *    (t, row, col) at index (t*h + row)*w + col.  vt_forward keeps tokens internally in
 *    2x2-block order (the four members of a merge group consecutive) and converts at
 *    its boundary, so every output documented here is in raster (or merged-raster)
 *    order.
 */
#ifndef VT_H_
#define VT_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define VT_API __attribute__((visibility("default")))
#else
#define VT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum vt_status {
  VT_OK = 0,
  VT_ERR_INVALID_ARG = 1, /* null pointer, non-positive or inconsistent size, misalignment */
  VT_ERR_SHAPE = 2,       /* image side not a multiple of patch*merge, wrong t, grid too large */
  VT_ERR_NOT_LOADED = 3,  /* forward before a complete vt_load_weights */
  VT_ERR_WEIGHT = 4,      /* missing, duplicate, unknown or wrong-shape weight */
  VT_ERR_WORKSPACE = 5,   /* workspace smaller than vt_workspace_bytes() */
  VT_ERR_UNSUPPORTED = 6, /* configuration outside what the kernels implement */
  VT_ERR_CUDA = 7,        /* a CUDA runtime call or launch failed */
  VT_ERR_TIMEOUT = 8      /* a kernel's bounded wait ran out (reported by vt_check) */
} vt_status;

/* Model configuration.  Source: "MiniMax-M3 Vision" model card, Architecture table
 * (layers, hidden, heads, intermediate, patch 14, temporal patch 2, 2x2 merge,
 * projector widths); "v2_loaders" findings, section 3 (rope_mode 3d, rope_theta
 * 10000).  The pages leave LayerNorm eps, the GELU form and the RoPE section split
 * open; the tower's workloads use eps 1e-6, GELU tanh and sections 16/32/32 (80) or
 * 8/12/12 (32). */
typedef struct vt_config {
  int layers;          /* tower depth (32) */
  int hidden;          /* tower width d (1280) */
  int heads;           /* attention heads H (16) */
  int head_dim;        /* D = hidden / heads (80); kernels support 32 and 80 */
  int mlp;             /* MLP width (5120) */
  int patch;           /* patch side (14) */
  int temporal_patch;  /* frames per patch; a still image repeats its frame (2) */
  int merge;           /* spatial merge side (2); only 2 is supported */
  int rope_sections[3];/* channels rotated by t, h, w; even, summing to head_dim */
  float rope_theta;    /* RoPE base (10000) */
  float ln_eps;        /* LayerNorm epsilon (1e-6) */
  int gelu_tanh;       /* tower MLP GELU: 1 = tanh form, 0 = erf form */
  int proj_gelu_tanh;  /* projector GELU form, same encoding */
  int proj_hidden;     /* projector width P (6144) */
  int proj_out;        /* projector output width (6144) */
  int use_rope;        /* 1 = apply 3D RoPE to q and k, 0 = no position encoding */
} vt_config;

/* One weight tensor, borrowed (not copied).  data: device bf16, dense row-major.
 * Names and shapes (d = hidden, m = mlp, P = proj_hidden, Po = proj_out):
 *   embeddings.proj.weight [d, 3, temporal_patch, patch, patch], embeddings.proj.bias [d]
 *   layers.{i}.ln1.weight/bias [d], layers.{i}.ln2.weight/bias [d]
 *   layers.{i}.attn.qkv.weight [3d, d] and .bias [3d]   (rows q | k | v), or
 *   layers.{i}.attn.{q,k,v}.weight [d, d] and .bias [d] (packed once by the library)
 *   layers.{i}.attn.o.weight [d, d], .bias [d]
 *   layers.{i}.mlp.fc1.weight [m, d], .bias [m]; layers.{i}.mlp.fc2.weight [d, m], .bias [d]
 *   proj.patch_fc1.weight [P, d], proj.patch_fc2.weight [P, P],
 *   proj.merge_fc1.weight [P, 4P], proj.merge_fc2.weight [Po, P], each with .bias
 * Linear weights are [out, in] as in PyTorch.  The qkv layout follows the ViTBlock of
 * "metrale_model_arch/weight_loader/qwen3_vl.rs" (load_vision_encoder: norm1, qkv,
 * proj, norm2, fc1, fc2 with biases). */
typedef struct vt_weight {
  const char* name;
  const void* data;
  int ndim;
  int64_t shape[5];
} vt_weight;

typedef struct vt_handle vt_handle;

/* Validates cfg and creates a handle.  Host only, no CUDA call.  Errors:
 * VT_ERR_INVALID_ARG for null pointers or non-positive sizes, heads*head_dim !=
 * hidden, odd sections or sections not summing to head_dim; VT_ERR_UNSUPPORTED for
 * merge != 2 or a head layout without a kernel. */
VT_API vt_status vt_create(const vt_config* cfg, vt_handle** out);

/* Frees the handle and the device memory it owns.  Synchronises the device.
 * Library-defined (the pages have no user API; this is the counterpart of dropping the
 * encoder that VisionEncoder::new of "spark_model/layers/vision_encoder/enc_impl/
 * init.rs" builds). */
VT_API vt_status vt_destroy(vt_handle* h);

/* Registers the n weights (all of them, in any order) on the current device, packs
 * separate q/k/v into a fused qkv weight, and uploads the RoPE cos/sin tables
 * (positions 0..4095 per axis, computed in double precision, stored fp32).
 * Synchronous.  Errors: VT_ERR_WEIGHT names the offending tensor in vt_last_error(). */
VT_API vt_status vt_load_weights(vt_handle* h, const vt_weight* w, int n);

/* Bytes of caller workspace vt_forward / vt_forward_video / vt_tower_layer /
 * vt_merge_project need for B images or clips of grid grid_thw (host int32[3] = t, h, w
 * in patches, t <= 4096).  Affine in B*t*h*w: no term grows with the square of the
 * sequence.  Host only.  Library-defined: it replaces the capacity policy of
 * "spark_model/layers/vision_encoder/enc_impl/init.rs" (derive_max_patches and the
 * [seq, seq] buffers of build_scratch) with a size that is linear in the tokens. */
VT_API vt_status vt_workspace_bytes(const vt_handle* h, int B, const int32_t* grid_thw, size_t* out);

/* Full forward: patch unfold -> patch embedding -> layers -> 2x2 merge -> projector.
 *   pixels    device fp32 [B, 3, H, W], already normalised, H = grid_h*patch, W = grid_w*patch
 *   grid_thw  host int32[3]; t must be 1 (clips: vt_forward_video); h and w even, <= 4096
 *   out       device bf16 [B, t*h*w/4, proj_out], merged tokens in raster (i, j) order
 *   tower_out device bf16 [B, t*h*w, hidden] in raster order, or NULL
 *   ws        device workspace of at least vt_workspace_bytes(h, B, grid_thw) bytes
 * Source: "MiniMax-M3 Vision" model card, Architecture table and notes (1280-wide tower
 * tokens, 5120-wide merged tokens, 6144-wide projected tokens). */
VT_API vt_status vt_forward(vt_handle* h, const float* pixels, const int32_t* grid_thw, int B, void* out,
                     void* tower_out, void* ws, size_t ws_bytes, void* stream);

/* vt_forward with HOST buffers: copies pixels (host fp32) to the device workspace,
 * runs the forward, copies out (host bf16 [B, N/4, proj_out]) back and synchronises
 * the stream.  pixels and out should be pinned for full copy speed.  Needs
 * vt_workspace_bytes(...) + B*3*H*W*4 + B*(N/4)*proj_out*2 bytes (rounded up to 256
 * each) of device workspace. */
VT_API vt_status vt_forward_host(vt_handle* h, const float* pixels_host, const int32_t* grid_thw, int B,
                          void* out_host, void* ws, size_t ws_bytes, void* stream);
VT_API vt_status vt_forward_host_workspace_bytes(const vt_handle* h, int B, const int32_t* grid_thw, size_t* out);

/* vt_forward_host without the final synchronisation: the copies and the forward are
 * enqueued on `stream` and the call returns.  out_host holds the result, and ws, the
 * pixels and out_host may be reused, only after the caller has synchronised the stream.
 * Calls on two streams with separate workspaces and output buffers overlap one batch's
 * copies with another batch's forward (a serving pipeline).  pixels_host and out_host
 * must be pinned for the copies to be asynchronous. */
VT_API vt_status vt_forward_host_async(vt_handle* h, const float* pixels_host, const int32_t* grid_thw, int B,
                                       void* out_host, void* ws, size_t ws_bytes, void* stream);

/* Video: B clips of `frames` frames each, all frames of one size.
 *   clips     device fp32 [B, frames, 3, H, W], already normalised
 *   frames    >= 1; temporal patch t takes frames t*tp .. t*tp+tp-1 (tp = the config's
 *             temporal_patch), the last frame repeated when frames is not a multiple of
 *             tp, so frames = 1 is vt_forward's still image
 *   grid_thw  host int32[3]; t must equal ceil(frames / tp); h and w as for vt_forward
 *   out       device bf16 [B, t*h*w/4, proj_out]: merged tokens in (t, i, j) raster order,
 *             the 2x2 merge within each temporal slice
 *   tower_out device bf16 [B, t*h*w, hidden] in (t, h, w) raster order, or NULL
 *   ws        device workspace of at least vt_workspace_bytes(h, B, grid_thw) bytes
 * All t*h*w tokens of a clip attend to each other; RoPE rotates by (t, h, w).  Errors:
 * VT_ERR_SHAPE when t does not match frames, as for vt_forward otherwise.  Source:
 * "MiniMax-M3 Vision" model card, Architecture table (Conv3d patch embed, temporal patch
 * size 2, 3D RoPE); the frame-repeat rule of the "v2_loaders" findings, section 3. */
VT_API vt_status vt_forward_video(vt_handle* h, const float* clips, int frames, const int32_t* grid_thw, int B,
                                  void* out, void* tower_out, void* ws, size_t ws_bytes, void* stream);

/* GPU preprocessing of decoded images: bicubic resize to the grid's size, scaling by
 * 1/255 and per-channel normalisation, x = (v/255 - mean[c]) / std[c].
 *   images    device uint8, the B images [H0_b, W0_b, 3] (RGB, rows of interleaved
 *             pixels, as decoded) concatenated in order; no alignment needed
 *   src_hw    host int32 [B, 2] = (H0_b, W0_b); each side at most 16x the target side
 *   grid_thw  host int32[3] = (1, h, w): every image is resized to h*patch x w*patch
 *   mean, std host float[3] each, or NULL for the OpenAI CLIP statistics
 *             (0.48145466, 0.4578275, 0.40821073) / (0.26862954, 0.26130258, 0.27577711)
 *   pixels    device fp32 [B, 3, h*patch, w*patch], the input vt_forward takes
 * The resize is cubic convolution with Keys' kernel (a = -0.5): output pixel centres map
 * onto input pixel centres, the kernel is stretched by the scale factor when shrinking
 * (every source pixel contributes), taps outside the image are dropped and the weights
 * renormalised; resized values are not clamped or rounded to 8 bits.  Needs no weights
 * (h may be unloaded).  Errors: VT_ERR_SHAPE for a grid t != 1 or a source side above 16x
 * the target, VT_ERR_INVALID_ARG for empty images or std <= 0.  Source: "v2_loaders"
 * findings, section 3 (bicubic resize to 672x672, OpenAI CLIP mean/std, patchify). */
VT_API vt_status vt_preprocess(const vt_handle* h, const uint8_t* images, const int32_t* src_hw, int B,
                               const int32_t* grid_thw, const float* mean, const float* std, float* pixels,
                               void* stream);

/* Full forward from decoded images: the preprocessing of vt_preprocess writes the patch
 * vectors of the patch-embedding GEMM directly (no fp32 pixel array), then the forward
 * of vt_forward.  Arguments as vt_preprocess and vt_forward; ws of at least
 * vt_workspace_bytes(h, B, grid_thw) bytes.  The result equals vt_forward applied to
 * vt_preprocess's pixels, bit for bit. */
VT_API vt_status vt_forward_u8(vt_handle* h, const uint8_t* images, const int32_t* src_hw, int B,
                               const int32_t* grid_thw, const float* mean, const float* std, void* out,
                               void* tower_out, void* ws, size_t ws_bytes, void* stream);

/* Variable-resolution batch: B images (1 <= B <= 64) of different patch grids in one
 * call, their tokens packed into one sequence; attention stays within each image.
 *   pixels  device fp32, the images' [3, H_b, W_b] arrays concatenated in order
 *           (H_b = grids[3b+1]*patch, W_b = grids[3b+2]*patch)
 *   grids   host int32 [B, 3] (t, h, w) per image; t = 1, h and w even, <= 4096
 *   out     device bf16 [sum_b N_b/4, proj_out]: image b's merged tokens (raster order)
 *           follow image b-1's
 *   tower_out  device bf16 [sum_b N_b, hidden] (raster order per image) or NULL
 *   ws      device workspace of vt_workspace_bytes_varlen(h, B, grids) bytes
 * Each image's result equals vt_forward on that image alone.  Source: the capacity
 * discussion of "spark_model/layers/vision_encoder/enc_impl/init.rs" (images of any
 * size up to a per-call bound share the encoder). */
VT_API vt_status vt_workspace_bytes_varlen(const vt_handle* h, int B, const int32_t* grids, size_t* out);
VT_API vt_status vt_forward_varlen(vt_handle* h, const float* pixels, const int32_t* grids, int B, void* out,
                                   void* tower_out, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- backward
 * Gradient of a scalar loss with respect to the pixels, given its gradient with
 * respect to the tower output: every layer backwards from the activations its forward saved,
 * then the patch embedding and the fold onto the image.  Weights are constants (no
 * weight gradients).  Source: "v2_loaders - Differentiable Vision Tower Loaders
 * (spark2)", summary and section 3 (the loaders are differentiable; the probe
 * backpropagates the pooled tower feature to the image); the forward differentiated is
 * that of the "MiniMax-M3 Vision" model card, Architecture table.  Still images only
 * (grid t = 1); head_dim 80 (RoPE 16/32/32) or 32 (8/12/12). */

/* Builds library-owned transposed copies of the tower weights (the size of the tower
 * weights again), after vt_load_weights; a later vt_load_weights drops them.
 * Synchronises the device.  VT_ERR_UNSUPPORTED for other head layouts. */
VT_API vt_status vt_enable_backward(vt_handle* h);

/* Bytes of the saved-activation buffer and of the workspace (which covers both
 * vt_forward_saved and vt_backward).  The saved buffer keeps, for every layer, what its
 * backward needs so that nothing is recomputed: the layer input, the rotated q and k,
 * v^T, the attention output and its per-query log-sum-exp, the residual stream after
 * attention and the MLP pre-activation (about (12*hidden + 2*mlp) bytes per token and
 * layer, 25.7 KB at the 1280/5120 tower).  Host only. */
VT_API vt_status vt_backward_bytes(const vt_handle* h, int B, const int32_t* grid_thw, size_t* saved_bytes,
                                   size_t* ws_bytes);

/* Forward of the tower that fills `saved` (device, opaque layout, vt_backward_bytes) and
 * writes the tower output tower_out (device bf16 [B, N, hidden], raster order).  pixels
 * as vt_forward; the arithmetic is vt_forward's. */
VT_API vt_status vt_forward_saved(vt_handle* h, const float* pixels, const int32_t* grid_thw, int B, void* tower_out,
                                  void* saved, size_t saved_bytes, void* ws, size_t ws_bytes, void* stream);

/* d_tower: device bf16 [B, N, hidden] (raster order), the loss gradient with respect to
 * the tower output of the vt_forward_saved call that filled `saved`; d_pixels: device
 * fp32 [B, 3, H, W], the loss gradient with respect to the pixels (the sum over the
 * temporal patch's two copies of each frame).  VT_ERR_NOT_LOADED before
 * vt_enable_backward. */
VT_API vt_status vt_backward(vt_handle* h, const void* saved, const int32_t* grid_thw, int B, const void* d_tower,
                             float* d_pixels, void* ws, size_t ws_bytes, void* stream);

/* One tower layer backward on raster-ordered tokens: dx = J^T dy for x_out = layer_i(x_in),
 * x_in, dy and dx device bf16 [B, h*w, hidden] (dx may equal dy).  Runs the layer's
 * forward with saved activations and its backward with the same kernels as
 * vt_forward_saved / vt_backward, so that a single layer of the tower's backward can be
 * checked on its own.  Workspace: vt_tower_layer_backward_bytes (it holds the one
 * layer's saved activations).  Still images (t = 1); VT_ERR_NOT_LOADED before
 * vt_enable_backward.  Source as for vt_backward; the layer is the ViTBlock of
 * "metrale_model_arch/weight_loader/qwen3_vl.rs". */
VT_API vt_status vt_tower_layer_backward_bytes(const vt_handle* h, int B, const int32_t* grid_thw, size_t* ws_bytes);
VT_API vt_status vt_tower_layer_backward(vt_handle* h, int layer, const void* x_in, const void* dy, void* dx,
                                         const int32_t* grid_thw, int B, void* ws, size_t ws_bytes, void* stream);

/* Attention backward alone, no rotary embedding: q, k, v device bf16 [B, H, N, D] (q, k
 * as the scores use them), dO device bf16 [B*N, H*D] (gradient of the output
 * [B, N, H, D]); writes dqkv device bf16 [B*N, 3*H*D] = [dq | dk | dv], each in the
 * [B*N, H*D] layout.  Recomputes the forward; no [N, N] buffer.  D in {32, 80}. */
VT_API vt_status vt_attention_backward_workspace_bytes(int B, int H, int N, int D, size_t* out);
VT_API vt_status vt_attention_backward(const void* q, const void* k, const void* v, const void* dO, void* dqkv, int B,
                                       int H, int N, int D, float scale, void* ws, size_t ws_bytes, void* stream);

/* LayerNorm backward plus a residual gradient: dx = dres + J^T dy for y = LN(x) (gamma);
 * all device bf16 [rows, cols] (gamma [cols]); dres may equal dx; cols a multiple of 8. */
VT_API vt_status vt_layernorm_backward(const void* x, const void* gamma, const void* dy, const void* dres, void* dx,
                                       int rows, int cols, float eps, void* stream);

/* One pre-LN tower layer i on raster-ordered tokens: x_out = layer_i(x_in), both
 * device bf16 [B, t*h*w, hidden]; x_in may equal x_out.  Source: ViTBlock of
 * "metrale_model_arch/weight_loader/qwen3_vl.rs" (norm1, qkv, proj, norm2, fc1, fc2);
 * model card Architecture (GELU, 3D RoPE). */
VT_API vt_status vt_tower_layer(vt_handle* h, int layer, const void* x_in, void* x_out, const int32_t* grid_thw,
                         int B, void* ws, size_t ws_bytes, void* stream);

/* Patch embedding alone for still images (t = 1): x = Conv3d(pixels) as [B, h*w, hidden]
 * bf16, raster order. */
VT_API vt_status vt_patch_embed(vt_handle* h, const float* pixels, const int32_t* grid_thw, int B, void* x_out,
                         void* ws, size_t ws_bytes, void* stream);

/* 2x2 merge + projector on raster-ordered tower tokens [B, t*h*w, hidden] (device bf16)
 * -> out [B, t*h*w/4, proj_out].  Source: model card, Architecture table (projector). */
VT_API vt_status vt_merge_project(vt_handle* h, const void* tower, const int32_t* grid_thw, int B, void* out,
                           void* ws, size_t ws_bytes, void* stream);

/* Bidirectional multi-head attention O_h = softmax(q_h k_h^T * scale) v_h, computed
 * tile by tile with an online softmax: no [N, N] buffer.  Source:
 * "spark_model/layers/vision_encoder/enc_impl/init.rs" (the ViT attention score
 * matrix per head; CEILING_MAX_PATCHES doc comment: larger images need tiled
 * attention).
 *   q, k, v  device bf16 [B, H, N, D];  o  device bf16 [B, N, H*D]
 *   pos_thw  device int32 [N, 3] token positions (t, h, w) for 3D RoPE of q and k, or
 *            NULL for none; sections / theta as in vt_config (ignored when NULL).  The
 *            rotation's cos and sin are single precision, taken of the angle after an
 *            exact double-precision reduction to within half a turn (a few 1e-7 off).
 *   scale    > 0, usually 1/sqrt(D)
 *   ws       device workspace of vt_attention_workspace_bytes() (rotated q, k and the
 *            transposed v): 3 * B*H*D*ceil8(N) * 2 bytes, linear in N.
 * D must be 32, 64, 80 or 96. */
VT_API vt_status vt_attention_workspace_bytes(int B, int H, int N, int D, size_t* out);
VT_API vt_status vt_attention(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int D,
                       const int32_t* pos_thw, const int32_t* sections, float theta, float scale, void* ws,
                       size_t ws_bytes, void* stream);

/* The attention kernel on operands already in its layout, no workspace:
 *   q, k device bf16 [B, H, N, D] (rotated if RoPE is wanted), vt device bf16
 *   [B, H, D, ld_vt] (v transposed, ld_vt >= N, multiple of 8), o [B, N, H*D]. */
VT_API vt_status vt_attention_prepared(const void* q, const void* k, const void* vt, int ld_vt, void* o, int B, int H,
                                int N, int D, float scale, void* stream);

/* vt_attention for callers that cannot allocate device memory, and so cannot pass a
 * workspace: for example code running inside a host framework whose allocator owns
 * all device memory, or a plugin interface that hands over only its input and output
 * buffers.  The pages describe no such entry point; it has no counterpart there.
 * Arguments and results are those of vt_attention without ws / ws_bytes.  Its scratch
 * (rotated q and k, transposed v) is a 32 MiB array compiled into the library, which
 * every GPU that loads libvt holds until the process exits; vt_attention_static_max_bytes
 * reports the size.  A problem needing more than that (3 * B*H*D*ceil8(N) * 2 bytes)
 * is rejected with VT_ERR_WORKSPACE before anything is launched.  Nothing is
 * allocated: no cudaMalloc, cudaFree or allocating library call.  The first call on
 * each device looks up the array's device address (cudaGetSymbolAddress) with that
 * device current; make that first call before any stream capture.  All calls share
 * the array and leave their contents in it; calls whose GPU work overlaps race on it
 * and must be serialised by the caller. */
VT_API vt_status vt_attention_static(const void* q, const void* k, const void* v, void* o, int B, int H, int N,
                                     int D, const int32_t* pos_thw, const int32_t* sections, float theta,
                                     float scale, void* stream);
VT_API vt_status vt_attention_static_max_bytes(size_t* out);

/* out[M, N] = act(A[M, K] W[N, K]^T + bias) + resid, bf16 in/out, fp32 accumulation on
 * the tensor cores.  bias [N] and resid [M, N] may be NULL; resid may equal out.
 * act: 0 none, 1 GELU tanh form, 2 GELU erf form.  N and K must be multiples of 8.
 * Every linear layer of the tower and projector has this form (model card,
 * Architecture table). */
VT_API vt_status vt_linear(const void* A, const void* W, const void* bias, const void* resid, void* out, int M, int N,
                    int K, int act, void* stream);
/* The same product with device scratch ws (ws_bytes >= vt_linear_workspace_bytes(),
 * 16-byte aligned) for a split-K tail: when M >= 1024 and the output tiles leave most
 * pairs of SMs idle in the last round of the grid, with K at least 2048, the K steps of
 * the remaining tiles are shared out and summed in fp32 by a second kernel in a fixed
 * order (the result does not depend on timing).  The forward uses this form for every
 * linear layer.  Library-defined; ws NULL or too small: runs as vt_linear. */
VT_API vt_status vt_linear_ws(const void* A, const void* W, const void* bias, const void* resid, void* out, int M,
                              int N, int K, int act, void* ws, size_t ws_bytes, void* stream);
/* Bytes of the split-K scratch (one 256 x 256 fp32 tile per pair of SMs).  Host only. */
VT_API vt_status vt_linear_workspace_bytes(size_t* out);

/* LayerNorm over rows: y = (x - mean) / sqrt(var + eps) * gamma + beta; x, y device
 * bf16 [rows, cols]; statistics in fp32 (CLIP-style pre-LN block). */
VT_API vt_status vt_layernorm(const void* x, const void* gamma, const void* beta, void* y, int rows, int cols,
                       float eps, void* stream);

/* Patch vectors of B images pixels [B, 3, H, W] (device fp32) -> out [B*gh*gw,
 * 3*tp*patch*patch] device bf16 (round to nearest even), in (c, t, kh, kw) order,
 * frame repeated tp times ("v2_loaders" findings, section 3).  order: 0 raster,
 * 1 2x2-block order. */
VT_API vt_status vt_patch_unfold(const float* pixels, void* out, int B, int H, int W, int patch, int temporal_patch,
                          int order, void* stream);

/* Host-only index maps of one grid (t, h, w), for exact comparison in tests:
 *   token_order [t*h*w]    raster index of the token at each position of 2x2-block order
 *   pos_thw     [t*h*w, 3] (t, row, col) of each raster token, the RoPE positions
 *   merge_src   [t*h*w/4, 4] raster indices gathered by each merged token, in the
 *               member order (0,0), (0,1), (1,0), (1,1)
 * Any output pointer may be NULL.  Library-defined debugging aid: it exposes the
 * readings of the 2x2 merge (model card, Architecture table) and of the 3D RoPE
 * positions ("v2_loaders" findings, section 3) for exact tests. */
VT_API vt_status vt_index_maps(const int32_t* grid_thw, int32_t* token_order, int32_t* pos_thw, int32_t* merge_src);

/* Synchronises the stream and reports device-side errors recorded by the kernels
 * (VT_ERR_TIMEOUT), clearing them, and pending launch errors (VT_ERR_CUDA).
 * Library-defined: the pages' loader checks extents only with a debug assertion that
 * release builds compile out (init.rs, build_scratch doc comment); here every wait is
 * bounded and its failure is reported through this call. */
VT_API vt_status vt_check(void* stream);

/* Diagnostic of the failure-detection path.  Launches one CTA whose only waiting
 * thread waits on an mbarrier that nothing arrives on; the wait is bounded like every
 * wait in the library's kernels, gives up after 1 s, records a device timeout and
 * returns.  The following vt_check() then returns VT_ERR_TIMEOUT (and clears it);
 * the CUDA context stays usable.  Nothing faults, traps or hangs. */
VT_API vt_status vt_selftest_wait_timeout(void* stream);

/* Message of the calling thread's last failed call ("" if none).  Library-defined.
 * Thread-local rather than per handle, because several entry points (vt_attention,
 * vt_linear, vt_layernorm, ...) take no handle. */
VT_API const char* vt_last_error(void);

/* Per-kernel-class device time of the calls made between vt_profile_begin and
 * vt_profile_end on one stream, measured with CUDA events around each launch.
 * Classes: 0 gemm, 1 attention, 2 layernorm, 3 patch unfold, 4 reorder, 5 attention
 * preparation.  vt_profile_read synchronises and returns, per class, the summed
 * milliseconds, kernel launch count (a linear layer with a split-K tail launches two
 * kernels) and algorithmic FLOPs (GEMM: 2MNK; attention: 4 N^2 D
 * per head and image) and bytes (memory-bound classes). */
VT_API vt_status vt_profile_begin(void* stream);
VT_API vt_status vt_profile_end(void* stream);
VT_API vt_status vt_profile_read(int cls, double* ms, int64_t* launches, double* flops, double* bytes);
/* The individual launches of the last profiled interval, in launch order:
 * vt_profile_launches returns their count (synchronising like vt_profile_read);
 * vt_profile_launch returns launch i's class, milliseconds, FLOPs and bytes. */
VT_API vt_status vt_profile_launches(int64_t* count);
VT_API vt_status vt_profile_launch(int64_t i, int* cls, double* ms, double* flops, double* bytes);

#ifdef __cplusplus
}
#endif

#endif /* VT_H_ */
