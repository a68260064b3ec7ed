/*
 * wd.h — C ABI of libwd, the B200 (sm_100a) denoising step of a Wan2.1-style
 * image-to-video DiT driven by a classifier-free-guided Euler flow-matching
 * sampler.
 *
 * Sources (cited by page title and section):
 *   [I2V] "图解 Wan2.1 I2V：从一张图到一段视频，模型到底发生了什么" (liyongzhi.xyz)
 *   [WAN] "Wan（通义万相）：大规模视频生成基础模型 — 技术深度解析 & Wan2.1 vs Wan2.2对比"
 *         (devpress.csdn.net)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers are DEVICE pointers (cudaMalloc'd or torch tensors) unless a
 *   comment says "host".  The caller owns every buffer; the library never
 *   allocates device memory.  Scratch comes from a caller-provided workspace
 *   whose size the *_bytes queries return.
 * - Tensors are dense, row-major, in the layouts written next to each
 *   argument.  Every device pointer must be 16-byte aligned, otherwise the
 *   call returns WD_ERR_ALIGN before launching anything.
 * - dtype: wd_dims.dtype selects the storage type of weight matrices and of
 *   activations handed between kernels: WD_F32 (float, all-fp32 SIMT path)
 *   or WD_BF16 (bfloat16 tensor-core path, fp32 accumulation).  Arguments
 *   typed `const void*` below have that type; `float*` arguments are always
 *   fp32 (residual stream, latents, biases, gains, modulation vectors).
 * - Calls are asynchronous on `stream` (a cudaStream_t).  Validation failures
 *   return before any launch; a failed launch returns WD_ERR_CUDA.  Device
 *   kernels never trap: bounded waits that run out set a device error word,
 *   which wd_check() reports as WD_ERR_TIMEOUT.
 * - No exception crosses the ABI.  wd_last_error() gives the calling thread's
 *   last message.
 */
#ifndef WD_H_
#define WD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* wd_stream; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  WD_OK = 0,
  WD_ERR_ARG = 1,         /* null pointer or bad scalar argument          */
  WD_ERR_SHAPE = 2,       /* dimensions the kernels do not support        */
  WD_ERR_DTYPE = 3,       /* unknown dtype                                */
  WD_ERR_ALIGN = 4,       /* a device pointer is not 16-byte aligned      */
  WD_ERR_WORKSPACE = 5,   /* workspace smaller than the *_bytes query     */
  WD_ERR_CUDA = 6,        /* CUDA launch or runtime error                 */
  WD_ERR_TIMEOUT = 7,     /* a bounded device wait ran out                */
  WD_ERR_UNSUPPORTED = 8  /* feature not built for this configuration     */
} wd_status;

/* WD_F16 (IEEE half) is not a model dtype: it names the cross-attention
 * operands of the WD_BF16 path (the K/V cache and the cross queries) and the
 * operand type accepted by wd_attention. */
typedef enum { WD_F32 = 0, WD_BF16 = 1, WD_F16 = 2 } wd_dtype;
typedef enum { WD_NORM_LAYER = 0, WD_NORM_RMS = 1 } wd_norm;

/* Model and video dimensions.  D = model width, heads x (D/heads) attention
 * heads, ffn = FFN hidden width, blocks = DiT blocks; T, H, W = latent frames,
 * height and width (H, W even); the token grid is T x H/2 x W/2 and the token
 * count L = T*(H/2)*(W/2) ([I2V] 5.1).  n_txt x c_txt text tokens (umT5,
 * [I2V] 3.1), n_img x c_img CLIP tokens ([I2V] 3.2).  n_img = 0 selects the
 * text-to-video model of [I2V] 9: 16 input channels (x_t alone, no y), no CLIP
 * projection, and a single-stream cross-attention over the text tokens only;
 * c_img and every image weight are then unused (may be 0 / NULL).  norm
 * selects the adaLN norm (LayerNorm without affine by default, [I2V] 5.2); eps
 * its epsilon. */
typedef struct {
  int D, heads, ffn, blocks;
  int T, H, W;
  int n_txt, c_txt, n_img, c_img;
  int dtype; /* wd_dtype */
  int norm;  /* wd_norm  */
  float eps;
} wd_dims;

/* Shared time MLP: e = t2(SiLU(t1(sin(tau)))), e0 = tp(SiLU(e)) ([I2V] 5.2).
 * All fp32.  t1_w [D,256], t2_w [D,D], tp_w [6D,D]; biases [D], [D], [6D]. */
typedef struct {
  const float *t1_w, *t1_b, *t2_w, *t2_b, *tp_w, *tp_b;
} wd_time_weights;

/* Text MLP (c_txt -> D -> D) and CLIP MLPProj (c_img -> D -> D), each
 * Linear -> GELU -> Linear ([I2V] 7 steps 1-2).  Matrices [out,in] in dtype. */
typedef struct {
  const void *txt1_w; const float *txt1_b; const void *txt2_w; const float *txt2_b;
  const void *img1_w; const float *img1_b; const void *img2_w; const float *img2_b;
} wd_ctx_weights;

/* One DiT block ([I2V] 5.2-5.5).  Matrices [out,in] in dtype, vectors fp32.
 *   qkv_w [3D,D] rows (q; k; v), qkv_b [3D]; g_q, g_k [D] QK-RMSNorm gains;
 *   o_w [D,D]; cn_g, cn_b [D] cross-attention pre-norm affine;
 *   cq_w, ck_w, cv_w (text K/V), cki_w, cvi_w (image K/V), co_w: [D,D];
 *   f1_w [ffn,D], f2_w [D,ffn]; mod [6,D] the block's modulation bias b_i
 *   ([WAN] 2.5), rows (shift1, scale1, gate1, shift2, scale2, gate2). */
typedef struct {
  const void *qkv_w; const float *qkv_b;
  const float *g_q, *g_k;
  const void *o_w; const float *o_b;
  const float *cn_g, *cn_b;
  const void *cq_w; const float *cq_b;
  const void *ck_w; const float *ck_b;
  const void *cv_w; const float *cv_b;
  const void *cki_w; const float *cki_b;
  const void *cvi_w; const float *cvi_b;
  const void *co_w; const float *co_b;
  const void *f1_w; const float *f1_b;
  const void *f2_w; const float *f2_b;
  const float *mod;
} wd_block_weights;

/* The six linear layers of one block quantised for the FP8 block
 * (wd_block_forward_fp8): e4m3 matrices [out, in] (one byte per element) and
 * their per-output-channel scales [out] fp32 from wd_quant_rows_e4m3, so that
 * W ~ scale[row] * q.  The biases, gains and modulation stay in
 * wd_block_weights. */
typedef struct {
  const void *qkv_q, *o_q, *cq_q, *co_q, *f1_q, *f2_q;
  const float *qkv_s, *o_s, *cq_s, *co_s, *f1_s, *f2_s;
  int attention_fp8;   /* 0: the block's self-attention in bf16; 1: the FP8 attention (wd_attention_fp8) */
} wd_block_weights_fp8;

/* Head ([I2V] 5.5): mod [2,D] (shift, scale biases added to e), w [64,D]
 * in dtype, b [64] fp32.  Output feature c*4 + kh*2 + kw. */
typedef struct {
  const float *mod;
  const void *w;
  const float *b;
} wd_head_weights;

/* ------------------------------------------------------------------ queries */
const char* wd_last_error(void);
const char* wd_version(void);

/* Synchronises `stream`, then reports any pending asynchronous CUDA error
 * (WD_ERR_CUDA) or a device wait that ran out (WD_ERR_TIMEOUT; the error
 * word is cleared by the call). */
wd_status wd_check(wd_stream stream);

/* Token count L = T*(H/2)*(W/2) ([I2V] 5.1), or 0 for invalid dims. */
int64_t wd_token_count(const wd_dims* d);

/* Workspace bytes that wd_patch_embed, wd_block_forward and wd_unpatchify
 * need for a batch of `batch` samples (one buffer serves all three). */
size_t wd_workspace_bytes(const wd_dims* d, int batch);

/* Bytes of the context buffer written by wd_context_embed:
 * ctx_txt [batch, n_txt, D] then ctx_img [n_img, D], dtype elements, plus
 * the MLP hidden scratch behind them. */
size_t wd_ctx_bytes(const wd_dims* d, int batch);

/* Bytes of ONE block's cross-attention K/V cache written by wd_cross_kv:
 * k_img [n_img,D], v_img [n_img,D], k_txt [batch,n_txt,D], v_txt [batch,n_txt,D]
 * in that order, each part starting on a 256-byte boundary.  Elements are
 * fp32 for WD_F32 and IEEE half for WD_BF16 (the text cross-attention softmax
 * is sharp, so its operands keep 11 significant bits rather than 8). */
size_t wd_kv_bytes(const wd_dims* d, int batch);

/* ------------------------------------------------------------------ the path */

/* Conditioning y = concat(mask, image latent) ([I2V] 4.1, Q3, Q6).
 * img_lat [16,T,H,W] fp32 -> y [20,T,H,W] fp32.  known_frames (HOST array of
 * n_known pixel-frame indices in [0, 4(T-1)]; NULL or n_known = 0 means {0})
 * marks the known frames; the mask channel c of latent frame f is 1 when
 * entry 4f+c of (frame 0 repeated 4 times, frames 1..F-1) is known. */
wd_status wd_build_cond_y(const wd_dims* d, const float* img_lat, const int* known_frames,
                          int n_known, float* y, wd_stream stream);

/* Text and CLIP projections, once per video ([I2V] 7 steps 1-2, 6).
 * txt [batch, n_txt, c_txt] and clip [n_img, c_img] in dtype (the CFG
 * unconditional row carries zeroed text, [I2V] Q5).  ctx receives
 * wd_ctx_bytes(d, batch) bytes: ctx_txt [batch,n_txt,D], ctx_img [n_img,D]
 * (dtype), then scratch.  With n_img = 0 there is no CLIP input (clip and the
 * img weights may be NULL). */
wd_status wd_context_embed(const wd_dims* d, const wd_ctx_weights* w, const void* txt,
                           const void* clip, int batch, void* ctx, wd_stream stream);

/* One block's cross-attention keys and values from the context written by
 * wd_context_embed ([I2V] 5.4: text uses Linear_k/Linear_v, image its own
 * k_img/v_img).  kv receives wd_kv_bytes(d, batch) bytes.  With n_img = 0
 * only the text keys and values are written (their parts start at 0). */
wd_status wd_cross_kv(const wd_dims* d, const wd_block_weights* w, const void* ctx, int batch,
                      void* kv, wd_stream stream);

/* Time modulation ([I2V] 5.2): tau (the noise level x 1000) -> e [D] and
 * e0 [6,D], both fp32. */
wd_status wd_time_mod(const wd_dims* d, const wd_time_weights* w, float tau, float* e, float* e0,
                      wd_stream stream);

/* Patch embedding of concat(x_t, y) ([I2V] 4.2, 5.1): Conv3d(36, D, (1,2,2),
 * stride (1,2,2)) as a GEMM.  x_t [batch,16,T,H,W] fp32, y [20,T,H,W] fp32
 * shared by the batch, w [D,144] (Conv3d weight [D,36,1,2,2] flattened) in
 * dtype, b [D] fp32 -> X [batch, L, D] fp32, token l = (f*(H/2)+y)*(W/2)+x.
 * Text-to-video (n_img = 0, [I2V] 9): Conv3d(16, D, ...) of x_t alone, w
 * [D,64], y unused (may be NULL). */
wd_status wd_patch_embed(const wd_dims* d, const float* x_t, const float* y, const void* w,
                         const float* b, int batch, float* X, void* ws, size_t ws_bytes,
                         wd_stream stream);

/* One DiT block, in place on the fp32 residual stream X [batch, L, D]
 * ([I2V] 5.2-5.5): adaLN-modulated full 3D self-attention with QK-RMSNorm and
 * 3D RoPE, gate1 residual; decoupled image/text cross-attention, plain
 * residual; adaLN-modulated GELU FFN, gate2 residual.  e0 [6,D] fp32 from
 * wd_time_mod; kv from wd_cross_kv for this block.  On the WD_BF16 path the
 * cross-attention queries are stored as IEEE half, like the K/V cache. */
wd_status wd_block_forward(const wd_dims* d, const wd_block_weights* w, const float* e0,
                           const void* kv, int batch, float* X, void* ws, size_t ws_bytes,
                           wd_stream stream);

/* The three pieces of wd_block_forward, callable one by one on the same
 * workspace (wd_workspace_bytes(d, batch) bytes), for sequence parallelism
 * (each GPU holds a slice of the tokens, [WAN] 5.2) and for the attention
 * cache (a later step reuses a block's attention output, [WAN] 5.3).  Run in
 * order on one token slice, wd_block_qkv (slice), wd_block_self_attention
 * (whole sequence) and wd_block_post (slice) give wd_block_forward's result
 * bit for bit: they launch the same kernels on the same rows.
 *
 * wd_block_qkv: for the n_tok tokens starting at token tok0 of the sequence
 * (0 <= tok0, tok0 + n_tok <= L) and every sample of the batch,
 * h = norm(X)(1 + scale1) + shift1, [q k v] = h Wqkv^T + b, then q, k <-
 * RoPE3D(RMSNorm_D(.) g) with each token's (frame, row, column) taken from
 * its place tok0 + i in the whole grid ([I2V] 5.2, 5.3 (1), (2)).
 * X [batch, n_tok, D] fp32 (read only); qkv [batch, n_tok, 3D] in dtype
 * (q, then k, then v of all heads).  The workspace serves as scratch. */
wd_status wd_block_qkv(const wd_dims* d, const wd_block_weights* w, const float* e0, int batch, int64_t tok0,
                       int64_t n_tok, const float* X, void* qkv, void* ws, size_t ws_bytes, wd_stream stream);

/* Full non-causal self-attention over the whole sequence for `heads` heads
 * (1 <= heads <= d->heads; fewer than all when the heads are split across
 * GPUs): qkv [batch, L, 3 * heads * dh] in dtype, laid out as q of the
 * heads, then k, then v; o [batch, L, heads * dh] in dtype ([I2V] 5.3). */
wd_status wd_block_self_attention(const wd_dims* d, int batch, int heads, const void* qkv, void* o, wd_stream stream);

/* The rest of the block for n_tok tokens of every sample (1 <= n_tok <= L):
 * X += gate1 (o Wo^T + b); X += Linear_co(decoupled cross-attention of
 * Linear_cq(LN_affine(X)) over kv); X += gate2 FFN(norm(X)(1 + scale2) +
 * shift2) ([I2V] 5.2-5.5).  o [batch, n_tok, D] in dtype (the attention
 * output of these tokens), X [batch, n_tok, D] fp32 in place. */
wd_status wd_block_post(const wd_dims* d, const wd_block_weights* w, const float* e0, const void* kv, int batch,
                        int64_t n_tok, const void* o, float* X, void* ws, size_t ws_bytes, wd_stream stream);

/* The block of wd_block_forward with its six linear layers on e4m3
 * operands ([WAN] 5.3: FP8 GEMM with per-token activation scales; here with
 * per-output-channel weight scales, w8).  Each GEMM input is quantised per
 * token row (scale = row amax / 448, codes rounded to nearest-even with
 * saturation, as wd_quant_rows_e4m3): the outputs of the three norms are
 * quantised from fp32 in the norm kernel, the attention outputs and the FFN
 * hidden (bf16) by the row quantiser.  The self- and cross-attention, QK-norm
 * + RoPE and the fp32 residual stream are those of the bf16 block.  WD_BF16
 * models with D and ffn multiples of 256 only (else WD_ERR_UNSUPPORTED /
 * WD_ERR_SHAPE).  ws: wd_workspace_bytes_fp8(d, batch) bytes.  With
 * w8->f2_q NULL the FFN's second layer stays bf16 (w->f2_w): the FFN hidden
 * is then not quantised, which saves its extra pass over the largest
 * activation of the block.  With w8->attention_fp8 the self-attention is the
 * FP8 attention of [WAN] 5.3 (wd_attention_fp8_quantize + wd_attention_fp8 on
 * the block's q, k, v). */
size_t wd_workspace_bytes_fp8(const wd_dims* d, int batch);
wd_status wd_block_forward_fp8(const wd_dims* d, const wd_block_weights* w, const wd_block_weights_fp8* w8,
                               const float* e0, const void* kv, int batch, float* X, void* ws, size_t ws_bytes,
                               wd_stream stream);

/* Head and unpatchify ([I2V] 5.5): z = LN(X)(1 + e + mod[1]) + e + mod[0],
 * p = z w^T + b, v[b,c,f,2y+kh,2x+kw] = p[b, l, c*4+kh*2+kw].
 * X [batch,L,D] fp32, e [D] fp32 -> v [batch,16,T,H,W] fp32. */
wd_status wd_unpatchify(const wd_dims* d, const wd_head_weights* w, const float* e, int batch,
                        const float* X, float* v, void* ws, size_t ws_bytes, wd_stream stream);

/* CFG-combined Euler step ([I2V] 7; [WAN] 2.7):
 * x[i] += dt * (v_uncond[i] + cfg_scale * (v_cond[i] - v_uncond[i])), or
 * x[i] += dt * v_cond[i] when v_uncond is NULL.  n fp32 elements.  x may
 * not overlap the velocities. */
wd_status wd_euler_cfg_step(float* x, const float* v_cond, const float* v_uncond, float cfg_scale,
                            float dt, size_t n, wd_stream stream);

/* ------------------------------------------------------------------ no-allocation variant
 * No counterpart in the source pages: an integration aid.  Some callers
 * cannot hand the library a workspace: code running inside a host framework
 * that owns the whole device memory pool and gives plug-ins no scratch, or a
 * latency-critical loop that must not call cudaMalloc (it can synchronise the
 * device and stall the other streams).  For them, wd_patch_embed_noalloc does
 * the work of wd_patch_embed with its patch-gather scratch in a fixed array of
 * this library, WD_NOALLOC_PATCH_SCRATCH_BYTES large, which every GPU that
 * loads the library reserves until the process exits.
 * - Same arguments and results as wd_patch_embed, minus the workspace.
 * - The scratch takes batch * L * K * element-size bytes, with K = 144 for
 *   the image-to-video model (36 channels x 2 x 2) and K = 64 for the
 *   text-to-video model (16 x 2 x 2): at most 174762 token rows in bf16 or
 *   87381 in fp32 for image-to-video, 393216 in bf16 or 196608 in fp32 for
 *   text-to-video.  Larger requests return WD_ERR_WORKSPACE before any
 *   launch.
 * - The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before capturing the stream into a graph.
 * - It allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * - Every call shares the one array, which keeps the last call's contents
 *   (each call overwrites all of the part it uses, so nothing needs
 *   clearing); calls that overlap on the GPU — on different streams, or
 *   from different threads — race on it and must be serialised by the
 *   caller. */
#define WD_NOALLOC_PATCH_SCRATCH_BYTES (48u << 20)
wd_status wd_patch_embed_noalloc(const wd_dims* d, const float* x_t, const float* y, const void* w,
                                 const float* b, int batch, float* X, wd_stream stream);

/* ------------------------------------------------------------------ building blocks
 * The kernels of the path, exposed one by one so that each can be checked on
 * its own.  Same conventions as above. */

/* C = epilogue(A B^T + bias) for A [M,K] and B [N,K] (a Linear weight), both
 * in `dtype` (wd_dtype), row-major with leading dimension K; bias [N] fp32 or
 * NULL.  epilogue 0: out [M,N] = v in dtype; 1: out = GELU(v) (erf form,
 * [I2V] 5.5; on the tensor cores the normal tail probability comes from
 * Abramowitz-Stegun 7.1.26, within 3.3e-7 of the exact GELU, on the CUDA
 * cores from erff) in dtype; 2: out = v in fp32; 3: out [M,N] fp32 += g*v with
 * g = gate_a + gate_b (either may be NULL; both NULL means 1) — the gated
 * residual of [I2V] 5.2; 5 (WD_BF16 only): out = v in IEEE half (the
 * cross-attention operands).  bf16 runs on the tcgen05 tensor cores (N a
 * multiple of 64, K a multiple of 8), fp32 on the CUDA cores. */
wd_status wd_gemm(int dtype, int M, int N, int K, const void* A, const void* B, const float* bias, int epilogue,
                  void* out, const float* gate_a, const float* gate_b, wd_stream stream);

/* Multi-head attention without mask ([I2V] 5.3, 5.4): for every batch b and
 * head h, o = softmax(q k1^T / sqrt(dh)) v1 [+ softmax(q k2^T / sqrt(dh)) v2].
 * q, o [batch, Lq, heads*dh]; k1, v1 [batch, n1, heads*dh] or, with
 * kv1_shared != 0, [n1, heads*dh] shared by the batch; k2/v2 likewise, or
 * NULL for one segment.  dh in {32, 64, 128}.  dtype WD_F32: all fp32;
 * WD_BF16: all bf16; WD_F16: q, k, v IEEE half and o bf16 (the bf16 path's
 * cross-attention).  The probabilities enter the P V product in the operand
 * type (bf16 or half), with fp32 softmax statistics and accumulation.
 * Kernels: bf16 and half with dh = 128 run on the tcgen05 tensor cores; bf16
 * and half with dh = 32 or 64, and every fp32 call, run on the CUDA cores
 * (a reference kernel, far slower).  A WD_BF16 model (wd_dims) with heads of
 * any width but 128 is refused with WD_ERR_UNSUPPORTED, so the model path
 * never takes the CUDA-core attention. */
wd_status wd_attention(int dtype, int batch, int Lq, int heads, int dh, const void* q, const void* k1, const void* v1,
                       int n1, int kv1_shared, const void* k2, const void* v2, int n2, int kv2_shared, void* o,
                       wd_stream stream);

/* The same attention for one key segment (k, v [batch or 1, n, heads*dh]),
 * also writing each row's log-sum-exp lse [batch, heads, Lq] fp32,
 * lse = log2 sum_j 2^(log2(e) q k_j^T / sqrt(dh)) (log2 units).  dtype WD_BF16
 * or WD_F32.  With it, attentions over disjoint parts of the keys can be
 * merged (wd_attention_merge): the ring level of the sequence parallelism of
 * [WAN] 5.2, where each GPU holds a part of the keys and values. */
wd_status wd_attention_lse(int dtype, int batch, int Lq, int heads, int dh, const void* q, const void* k, const void* v,
                           int n, int kv_shared, void* o, float* lse, wd_stream stream);

/* Merges one part's attention into a running result: o_run [batch, Lq,
 * heads*dh] and lse_run [batch, heads, Lq] (fp32, updated in place) absorb
 * o_part (dtype: WD_BF16 or WD_F32) and lse_part from wd_attention_lse over a
 * disjoint set of keys: with M = max(lse_run, lse_part), a = 2^(lse_run - M),
 * c = 2^(lse_part - M): o_run = (a o_run + c o_part) / (a + c), lse_run =
 * M + log2(a + c).  first != 0: o_run and lse_run are set to the part (their
 * old contents are not read).  out (optional, dtype, same layout as o_part)
 * receives the merged output rounded to dtype. */
wd_status wd_attention_merge(int dtype, int batch, int Lq, int heads, int dh, float* o_run, float* lse_run,
                             const void* o_part, const float* lse_part, int first, void* out, wd_stream stream);

/* FP8 attention ([WAN] 5.3, "FlashAttention3 FP8": the Q/K inner product in
 * INT8, O = P V in FP8, accumulation across key blocks in FP32), non-causal,
 * one key segment, head dim 128, bf16 q, k, v and output.
 *
 * Operands, in one device buffer laid out by wd_attention_fp8_layout (byte
 * offsets, each 256-byte aligned; the buffer itself 256-byte aligned):
 *   q8  int8 [batch, Lq, heads*128], one scale per (row, head): sq [batch, heads, Lq]
 *   k8  int8 [batch, Lk, heads*128], one scale per (128-key block, head): sk [batch, heads, ceil(Lk/128)]
 *   v8t e4m3 [batch, heads, 128, lkp] (V transposed: keys contiguous; lkp = Lk rounded up to 16,
 *       keys Lk..lkp zero), one scale per (channel, head, batch): sv [batch, heads*128]
 *   v_amax scratch [batch, heads*128]
 * Scales: int8 amax/127, e4m3 amax/448 (fp32, IEEE division; 1 for an all-zero
 * row, block or channel); codes: round to nearest even (int8 clamped to
 * +-127; e4m3 saturating at +-448).
 * Attention: per 128-key block, S = q8 k8^T exactly (int32), logits
 * t = S sq sk log2(e)/sqrt(128) (log2 units), the online softmax with a lazy
 * reference max m (moved to the block's row max only when that exceeds m by
 * more than 8; the running O and l are then scaled by 2^(m_old - m)),
 * p = 2^(t - m) rounded to e4m3 for O += P8 v8 (fp32 accumulation) while l
 * sums the unrounded p; out = O sv / l rounded to bf16.  The result depends on
 * that reference within e4m3 precision of P (the oracle follows the same
 * blocks and rule).
 * Errors: dh != 128 -> WD_ERR_UNSUPPORTED; empty shapes, Lq or Lk above 2^30 ->
 * WD_ERR_SHAPE; a buffer smaller than layout.bytes -> WD_ERR_WORKSPACE;
 * misaligned pointers or strides -> WD_ERR_ALIGN. */
typedef struct {
  size_t q8, sq, k8, sk, v8t, sv, v_amax;   /* byte offsets in the buffer */
  size_t bytes;                             /* the buffer's size */
  int64_t lkp;                              /* keys per V^T row */
} wd_attn_fp8_layout;
wd_status wd_attention_fp8_layout(int batch, int64_t Lq, int64_t Lk, int heads, int dh, wd_attn_fp8_layout* out);

/* Quantises q [batch, Lq, heads*dh] (row stride q_rs elements; 8-byte aligned)
 * and k, v [batch, Lk, heads*dh] (row stride kv_rs; k 8-byte, v 16-byte
 * aligned; strides multiples of 8) into buf (two kernels and a memset, on
 * stream).  q, k, v may be the column blocks of one fused q|k|v buffer. */
wd_status wd_attention_fp8_quantize(int batch, int64_t Lq, int64_t Lk, int heads, int dh, const void* q, int64_t q_rs,
                                    const void* k, const void* v, int64_t kv_rs, void* buf, size_t buf_bytes,
                                    wd_stream stream);

/* The attention on the quantised operands in buf (from
 * wd_attention_fp8_quantize with the same shape): o [batch, Lq, heads*dh]
 * bf16, row stride o_rs elements (16-byte aligned, a multiple of 8). */
wd_status wd_attention_fp8(int batch, int64_t Lq, int64_t Lk, int heads, int dh, const void* buf, size_t buf_bytes,
                           void* o, int64_t o_rs, wd_stream stream);

/* FP8 GEMM building blocks ([WAN] 5.3: FP8 GEMM with per-token activation and
 * per-channel weight scales), used by wd_block_forward_fp8 and exposed to be
 * checked and measured on their own. */

/* Per-row e4m3 quantisation: for each row r of x [rows, K] (dtype WD_BF16 or
 * WD_F32, K a multiple of 8), scale[r] = max_k |x[r,k]| / 448 (1 for an
 * all-zero row, fp32, IEEE division) and q[r,k] = e4m3(x[r,k] / scale[r])
 * (one byte per element, round-to-nearest-even, saturating at +-448), so that
 * x ~ scale[r] * q.  For a Linear weight [out, in] the rows are the output
 * channels. */
wd_status wd_quant_rows_e4m3(int dtype, int rows, int K, const void* x, void* q, float* scale, wd_stream stream);

/* FP8 GEMM on the tcgen05 tensor cores (kind::f8f6f4): with
 * v[m,n] = sa[m] * sb[n] * sum_k Aq[m,k] Bq[n,k] + bias[n] (fp32 accumulation),
 * the epilogues of wd_gemm: 0 out bf16 = v, 1 out bf16 = GELU(v), 2 out fp32
 * = v, 3 out fp32 += (gate_a + gate_b) * v.  Aq [M,K] and Bq [N,K] e4m3 from
 * wd_quant_rows_e4m3, sa [M], sb [N] their scales; N a multiple of 256, K a
 * multiple of 16; out [M,N].  Epilogue 5 (out IEEE half = v) as for wd_gemm. */
wd_status wd_gemm_fp8(int M, int N, int K, const void* Aq, const float* sa, const void* Bq, const float* sb,
                      const float* bias, int epilogue, void* out, const float* gate_a, const float* gate_b,
                      wd_stream stream);

/* ------------------------------------------------------------------ test hooks
 * Two entry points that exist only so that tests can reach pieces of the
 * kernels no output of the path exposes on its own.  Not part of the step. */

/* Evaluates, for each of the n fp32 values x[i], the 2^x of the attention
 * kernels' world: y_fma[i] = the FMA-pipe 2^x that the softmax of the
 * tensor-core attention uses for some of its exponentials (range reduction
 * to x = j + f, |f| <= 1/2, a degree-3 polynomial in f with a stated relative
 * error below 7.5e-5, inputs below -125 clamped to -125); y_fma2[i] = the
 * same function in its packed two-lane form (f32x2 instructions), evaluated
 * on the pair (x[i], x[i^1]), which must equal y_fma[i]; y_mufu[i] = the MUFU
 * approximation ex2.approx.ftz.f32 used for the rest; y_lib[i] = CUDA's
 * exp2f.  All device arrays of n floats; n > 0. */
wd_status wd_test_exp2(const float* x, float* y_fma, float* y_fma2, float* y_mufu, float* y_lib, int64_t n,
                       wd_stream stream);

/* Evaluates, for each of the n fp32 values x[i], the two GELUs of the library:
 * y_as[i] = the tensor-core GEMM epilogue's x * Phi(x), with the normal tail
 * probability from the rational approximation 7.1.26 of Abramowitz and Stegun
 * (erf within 1.5e-7), a MUFU reciprocal and a MUFU 2^x; y_as2[i] = the same
 * function in its packed two-lane form (f32x2 instructions, the one the
 * epilogue runs), evaluated on the pair (x[i], x[i^1]), which must equal
 * y_as[i]; y_erf[i] = the CUDA-core path's 0.5 x (1 + erff(x / sqrt 2)).
 * All device arrays of n floats; n > 0. */
wd_status wd_test_gelu(const float* x, float* y_as, float* y_as2, float* y_erf, int64_t n, wd_stream stream);

/* Launches one warp that waits on an mbarrier phase nothing completes, with
 * the library's bounded wait given a limit of limit_ns (at most 100 ms, not
 * the pipelines' 2 s).  When the limit runs out the wait records `site`
 * (non-zero) in the device error word and the kernel returns; out[0] (device
 * int) receives 1 if the wait saw completion, 0 if it ran out.  A following
 * wd_check(stream) then returns WD_ERR_TIMEOUT naming the site and clears
 * the word, as it does for a pipeline wait that ran out. */
wd_status wd_test_wait_timeout(uint64_t limit_ns, unsigned site, int* out, wd_stream stream);

/* ------------------------------------------------------------------ tracing
 * Every kernel launch is counted by class.  With timing enabled, each launch
 * is also bracketed by two CUDA events recorded on its own stream, so the
 * device time of each class can be read for any region of work. */
typedef enum {
  WD_KC_GEMM = 0, WD_KC_ATTN_SELF = 1, WD_KC_ATTN_CROSS = 2, WD_KC_NORM = 3, WD_KC_ROPE = 4,
  WD_KC_EULER = 5, WD_KC_SMALL = 6, WD_KC_COUNT = 7
} wd_kernel_class;
void wd_trace_enable(int on);
/* Waits for the recorded events, writes per-class launch counts and summed
 * device milliseconds since the previous read (either array may be NULL;
 * both have WD_KC_COUNT entries), then starts a new region. */
wd_status wd_trace_read(int64_t* launches, double* total_ms);

/* Debugging aid: bit 0 routes bf16 GEMMs, bit 1 bf16 attention, to the
 * CUDA-core kernels instead of the tensor-core ones.  Process-wide, for
 * tests only: while a bit is set every call of the library runs at CUDA-core
 * speed.  wd_debug_flags() returns the bits in force (0 by default). */
void wd_set_debug_flags(unsigned flags);
unsigned wd_debug_flags(void);

#ifdef __cplusplus
}
#endif
#endif /* WD_H_ */
