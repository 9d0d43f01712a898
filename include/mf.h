/*
 * mf.h -- C ABI of libmf, the B200 (sm_100a) packed joint-attention block.
 *
 * The block is the data-parallel hot path of the Mage-Flow NR-MMDiT backbone:
 * image-latent token grids and text tokens of several samples share one flat
 * token buffer (a "pack"), delimited by per-sample cumulative offsets. One
 * block forward runs modality-specific adaptive LayerNorm modulation, per-sample
 * 2D RoPE (3D with a frame axis for edit packs) on Q and K, block-diagonal
 * variable-length softmax attention and a gated residual.
 *
 * Sources (page title, then section); the pages describe the operations in
 * words only:
 *   [pack] picx.dev "Mage-Flow" summary, Methodology > Native-Resolution MMDiT
 *          (NR-MMDiT), "Native-resolution packing": variable-length latent and
 *          text sequences packed under a fixed token budget, attention run with
 *          per-sample cumulative offsets.
 *   [rope] gist.science "Resumo Tecnico: Mage-Flow", Metodologia > 2. NR-MMDiT,
 *          "Empacotamento de Resolucao Nativa": per-sample 2D rotary embeddings.
 *   [edit] picx.dev summary, Methodology > NR-MMDiT, "Conditioning": source and
 *          target latents concatenated under a 3D RoPE with a frame dimension.
 *   [norm] picx.dev summary, Methodology > NR-MMDiT: modality-specific
 *          normalization and joint self-attention.
 *   [fuse] picx.dev summary, Methodology > Training Infrastructure: fused
 *          adaptive normalization / RoPE / gating in NR-MMDiT.
 *   [cfg]  picx.dev summary, Methodology > NR-MMDiT, "Packed CFG inference":
 *          the conditional and unconditional branches packed into one forward.
 *   [train] picx.dev summary, Methodology > Training Infrastructure and
 *          Table 4: the packed NR-MMDiT is trained (MFU and training speedup),
 *          so each training step also runs the backward of the block.
 *   [vae]  picx.dev summary, Methodology > Mage-VAE, "Architecture": a fully
 *          convolutional one-step diffusion decoder (and its dual encoder) of
 *          stacked convolutional blocks; 16x downsampled, 128-channel latents.
 *   [vfuse] picx.dev summary, Methodology > Training Infrastructure: the
 *          normalization - activation - residual chains of the VAE's repeated
 *          blocks run as fused CUDA kernels.
 * Where the pages are silent the library follows one stated reading: RoPE
 * splits head_dim evenly across the axes in whole adjacent-channel pairs, base
 * 10000 by default, leftover channels unrotated; text token j of a sample sits
 * at position max(grid_h, grid_w) + j on every axis; LayerNorm has no affine
 * parameters; x_mod = LN(x) * (1 + scale) + shift; y = x + gate * attn.
 *
 * Conventions for every entry point:
 *   - Tensors are dense, row-major, in device memory unless marked "host".
 *     bf16 tensors are passed as mf_bf16 (the 16-bit pattern of a bfloat16).
 *   - The caller owns and allocates all memory; the library never allocates
 *     device memory. Scratch space is passed as (workspace, ws_bytes).
 *   - Device pointers must be 16-byte aligned.
 *   - Argument errors return MF_ERR_INVALID (or MF_ERR_UNSUPPORTED for shapes
 *     outside the supported set) before anything is launched.
 *   - Work is enqueued asynchronously on `stream`. A failure detected inside a
 *     kernel (a bounded wait that ran out, an id out of range in device data)
 *     is recorded in a per-device error word; mf_get_error() reports it.
 *   - Supported shapes: head_dim D in {64, 128}; hid = H * D with H <= 128 and
 *     hid <= 4096; S <= MF_MAX_SAMPLES; T < 2^24.
 */
#ifndef MF_H_
#define MF_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MF_ABI_VERSION 1
#define MF_MAX_SAMPLES 512
#define MF_MAX_TOKENS (1 << 24)

typedef uint16_t mf_bf16; /* bfloat16 bit pattern */

typedef enum {
  MF_OK = 0,
  MF_ERR_INVALID = 1,     /* bad argument, or bad id found in device data */
  MF_ERR_CUDA = 2,        /* a CUDA runtime call failed */
  MF_ERR_TIMEOUT = 3,     /* a bounded device-side wait ran out */
  MF_ERR_UNSUPPORTED = 4  /* valid but outside the supported shapes */
} mf_status;

/* One sample of a pack: `frames` latent grids of grid_h x grid_w tokens (frame
 * major, then row major), then n_text text tokens. frames is 0 (a text-only
 * segment), 1, or 2 (source + target of an edit; 3D RoPE only). is_dummy marks
 * the padding segment of a training pack; the library computes it like any other
 * sample (it only matters to FLOP accounting). */
typedef struct {
  int32_t frames;
  int32_t grid_h;
  int32_t grid_w;
  int32_t n_text;
  int32_t is_dummy;
} mf_sample_desc;

int32_t mf_abi_version(void);
const char* mf_status_string(mf_status s);

/* Text of the last CUDA runtime error a call on this host thread turned into
 * MF_ERR_CUDA ("" if none). The string belongs to the library and stays valid
 * until the next failing call on this thread. */
const char* mf_last_error_detail(void);

/* Pack metadata [pack], [rope], [edit].
 * desc: host array of S descriptors. rope_axes: 2 (h, w) or 3 (f, h, w).
 * budget: token budget (0 = none); T > budget is MF_ERR_INVALID.
 * Outputs: cu_seqlens_h (host, S+1 int32, exclusive prefix sum of sample
 * lengths), *T_out (host), and on the device cu_seqlens_d [S+1] int32,
 * pos_ids_d [T][3] int32 (frame, h, w), tok_sample_d [T] int32 (sample of each
 * token), tok_mod_d [T] uint8 (0 = image latent, 1 = text).
 * If all four device pointers are NULL only the host outputs are written (a
 * size query). Image token (f, h, w) has position (f, h, w) (f = 0 in 2D
 * packs); text token j has (p, p, p) with p = max(grid_h, grid_w) + j. */
mf_status mf_pack_build(const mf_sample_desc* desc, int32_t S, int32_t rope_axes,
                        int32_t budget, int32_t* cu_seqlens_h, int32_t* cu_seqlens_d,
                        int32_t* pos_ids_d, int32_t* tok_sample_d, uint8_t* tok_mod_d,
                        int32_t* T_out, cudaStream_t stream);

/* Modulation vectors [norm], [fuse]: mod[s][m][j][i] =
 * sum_c c[s][c] * W[c][(3m + j) * hid + i], m in {image, text},
 * j in {shift, scale, gate}. c: [S][C] fp32, W: [C][6*hid] fp32,
 * mod: [S][2][3][hid] fp32 (written). fp32 accumulation in c order. */
mf_status mf_adaln_params(const float* c, const float* W, int32_t S, int32_t C,
                          int32_t hid, float* mod, cudaStream_t stream);

/* Modality-specific adaLN [norm]: x_mod[t] = LN(x[t]) * (1 + scale[s,m]) +
 * shift[s,m], LN without affine parameters, population variance, eps given.
 * x, x_mod: [T][hid] bf16 (must not alias); mod from mf_adaln_params;
 * tok_sample / tok_mod from mf_pack_build. A tok_sample outside [0, S) is
 * recorded as MF_ERR_INVALID and that row is left unwritten. hid % 8 == 0. */
mf_status mf_adaln_modulate(const mf_bf16* x, const float* mod, const int32_t* tok_sample,
                            const uint8_t* tok_mod, int32_t T, int32_t S, int32_t hid,
                            float eps, mf_bf16* x_mod, cudaStream_t stream);

/* Per-sample RoPE on Q and K [rope], [edit]. q, k: [T][H][D] bf16; either may be
 * NULL to skip it. q_out / k_out may equal q / k (in place). Channel pairs
 * (2i, 2i+1) of the chunk of axis a (width d_a = 2 * floor(D / (2*rope_axes)),
 * chunks in axis order (h, w) or (f, h, w)) turn by pos_a * base^(-2i / d_a);
 * channels past the last chunk are copied. fp32 arithmetic, bf16 output. */
mf_status mf_rope_apply(const mf_bf16* q, const mf_bf16* k, const int32_t* pos_ids,
                        int32_t T, int32_t H, int32_t D, int32_t rope_axes, float base,
                        mf_bf16* q_out, mf_bf16* k_out, cudaStream_t stream);

/* Backward of mf_rope_apply [rope], [train]: every pair rotation is orthogonal,
 * so the gradient turns back by the same angle (the transpose):
 * dx0 = c g0 + s g1, dx1 = -s g0 + c g1 for the output gradient (g0, g1) of a
 * pair; unrotated channels are copied. Same arguments, layout, aliasing and
 * checks as mf_rope_apply (dq_r / dk_r in, dq / dk out). */
mf_status mf_rope_bwd(const mf_bf16* dq_r, const mf_bf16* dk_r, const int32_t* pos_ids,
                      int32_t T, int32_t H, int32_t D, int32_t rope_axes, float base,
                      mf_bf16* dq, mf_bf16* dk, cudaStream_t stream);

/* Block-diagonal varlen attention [pack], [norm]: for every sample s and head h,
 * O = softmax(Q K^T * softmax_scale) V over the sample's own tokens only.
 * q, k, v, o: [T][H][D] bf16 (o must not alias inputs). cu_seqlens_d and
 * cu_seqlens_h: the same S+1 offsets on device and host; T = cu_seqlens_h[S].
 * pos_ids: NULL when q and k are already rotated, else [T][3] and RoPE with
 * (rope_axes, base) is applied to q and k first (needs workspace).
 * softmax_scale: finite and > 0 (the usual choice is 1/sqrt(D)).
 * lse: NULL or [H][T] fp32, natural-log log-sum-exp of each row's scores.
 * workspace: ws_bytes >= mf_workspace_size(T, H, D, pos_ids != NULL).
 * QK^T and PV run on tcgen05 tensor cores, bf16 operands, fp32 accumulation;
 * P is rounded to bf16 for PV. */
mf_status mf_varlen_attn_fwd(const mf_bf16* q, const mf_bf16* k, const mf_bf16* v,
                             const int32_t* cu_seqlens_d, const int32_t* cu_seqlens_h,
                             int32_t S, int32_t H, int32_t D, float softmax_scale,
                             const int32_t* pos_ids, int32_t rope_axes, float base,
                             mf_bf16* o, float* lse, void* workspace, size_t ws_bytes,
                             cudaStream_t stream);

/* Backward of mf_varlen_attn_fwd [pack], [train] (q and k as the attention saw
 * them, i.e. already rotated): for every sample s and head h, with
 * P = softmax(scale Q K^T) rebuilt from lse,
 *   dV = P^T dO, dP = dO V^T, dS = P * (dP - rowsum(dO * O)),
 *   dQ = scale dS K, dK = scale dS^T Q;
 * nothing crosses a sample boundary. q, k, v, o, d_o: [T][H][D] bf16 (o the
 * forward's output, d_o the loss gradient with respect to it); lse: [H][T] fp32,
 * the forward's natural-log log-sum-exp. dq, dk, dv: [T][H][D] bf16 outputs,
 * disjoint from every input and from each other. Offsets, S, H, D and
 * softmax_scale as for the forward (cu_seqlens_d must hold the same offsets as
 * cu_seqlens_h; the backward's kernels take the pack geometry from the host
 * copy). workspace (fp32 dQ accumulator and row
 * tables): ws_bytes >= mf_attn_bwd_workspace_size(T, S, H, D), disjoint from
 * everything else. The five products run on tcgen05 tensor cores with bf16
 * operands and fp32 accumulation; P and dS are rounded to bf16 as operands. */
mf_status mf_varlen_attn_bwd(const mf_bf16* q, const mf_bf16* k, const mf_bf16* v,
                             const mf_bf16* o, const mf_bf16* d_o, const float* lse,
                             const int32_t* cu_seqlens_d, const int32_t* cu_seqlens_h,
                             int32_t S, int32_t H, int32_t D, float softmax_scale,
                             mf_bf16* dq, mf_bf16* dk, mf_bf16* dv, void* workspace,
                             size_t ws_bytes, cudaStream_t stream);
size_t mf_attn_bwd_workspace_size(int32_t T, int32_t S, int32_t H, int32_t D);

/* Backward of mf_adaln_params [norm], [train]: with mod = c W (mod flattened to
 * [S][6*hid]), dW = c^T dmod and dc = dmod W^T. dmod: [S][2][3][hid] fp32, the
 * gradient of the modulation vectors (the shift, scale and gate slots that
 * mf_adaln_modulate_bwd and mf_gated_residual_bwd write); c: [S][C] and
 * W: [C][6*hid] fp32 as in the forward. Outputs, either of which may be NULL
 * (not both): dc [S][C] fp32 and dW [C][6*hid] fp32, overwritten, disjoint from
 * every input and from each other. Same shape limits as mf_adaln_params. fp32
 * arithmetic; every sum is taken in a fixed order (no atomics), so repeated
 * calls give the same bits. */
mf_status mf_adaln_params_bwd(const float* dmod, const float* c, const float* W, int32_t S,
                              int32_t C, int32_t hid, float* dc, float* dW, cudaStream_t stream);

/* Gated residual [fuse]: y[t] = x[t] + gate[s,m] * o[t], o viewed as [T][H*D].
 * x, o, y: [T][hid] bf16 (y may equal x). Same id checks as mf_adaln_modulate. */
mf_status mf_gated_residual(const mf_bf16* x, const mf_bf16* o, const float* mod,
                            const int32_t* tok_sample, const uint8_t* tok_mod, int32_t T,
                            int32_t S, int32_t hid, mf_bf16* y, cudaStream_t stream);

/* Backward of mf_gated_residual [fuse], [train]: for y = x + gate[s,m] * o,
 * d_o = gate[s,m] * dy and dmod[s][m][gate][:] = the sum over the tokens of
 * sample s and modality m of dy * o (dx = dy is the caller's identity path).
 * dy, o, d_o: [T][hid] bf16 (d_o may equal dy; it must not overlap o). dmod:
 * [S][2][3][hid] fp32; only its gate slots are written (overwritten, zero for a
 * (sample, modality) without tokens). Sums use fp32 atomics (their order, and so
 * the last bits, can vary between runs). Bad ids as for mf_gated_residual. */
mf_status mf_gated_residual_bwd(const mf_bf16* dy, const mf_bf16* o, const float* mod,
                                const int32_t* tok_sample, const uint8_t* tok_mod, int32_t T,
                                int32_t S, int32_t hid, mf_bf16* d_o, float* dmod,
                                cudaStream_t stream);

/* Backward of mf_adaln_modulate [norm], [train]: with xhat = (x - mean) * rstd
 * over each row, g = dx_mod * (1 + scale[s,m]):
 *   dx = resid + (g - mean(g) - xhat * mean(g * xhat)) * rstd,
 *   dmod[s][m][shift][:] = sum dx_mod, dmod[s][m][scale][:] = sum dx_mod * xhat
 * (sums over the tokens of sample s and modality m). dx_mod, x, dx and resid:
 * [T][hid] bf16; resid may be NULL (taken as 0) and dx may equal resid (in
 * place); dx must not overlap x, dx_mod, dmod or the workspace. dmod: only its
 * shift and scale slots are written (overwritten). eps as in the forward.
 * workspace: ws_bytes >= mf_adaln_bwd_workspace_size(T) (row statistics). */
mf_status mf_adaln_modulate_bwd(const mf_bf16* dx_mod, const mf_bf16* x, const float* mod,
                                const int32_t* tok_sample, const uint8_t* tok_mod,
                                const mf_bf16* resid, int32_t T, int32_t S, int32_t hid,
                                float eps, mf_bf16* dx, float* dmod, void* workspace,
                                size_t ws_bytes, cudaStream_t stream);
size_t mf_adaln_bwd_workspace_size(int32_t T);

/* The whole block [fuse]: x_mod = adaLN(x); then RoPE on q and k, varlen
 * attention with softmax scale 1/sqrt(D), and the gated residual fused into the
 * attention epilogue: y = x + gate * O (O never reaches memory).
 * x, x_mod, y: [T][hid] bf16; q, k, v: [T][H][D] bf16; mod, ids and offsets as
 * above. workspace: ws_bytes >= mf_workspace_size(T, H, D, 1). */
mf_status mf_block_fwd(const mf_bf16* x, const mf_bf16* q, const mf_bf16* k, const mf_bf16* v,
                       const float* mod, const int32_t* cu_seqlens_d,
                       const int32_t* cu_seqlens_h, const int32_t* pos_ids,
                       const int32_t* tok_sample, const uint8_t* tok_mod, int32_t S, int32_t H,
                       int32_t D, int32_t rope_axes, float base, float eps, mf_bf16* x_mod,
                       mf_bf16* y, void* workspace, size_t ws_bytes, cudaStream_t stream);

/* mf_block_fwd without a workspace argument, for callers that cannot allocate
 * device memory (for example a plugin inside a host application that owns all
 * device memory and gives it no allocator, or a caller that must not make a call
 * which can synchronise the device). The paper has no counterpart: this is a
 * library convenience. Arguments and results are those of mf_block_fwd; the
 * workspace mf_block_fwd would take (the fused RoPE's (cos, sin) table and the
 * rotated k) is a file-scope device array of MF_NOALLOC_SCRATCH_BYTES that every
 * GPU loading the library holds until exit, so a pack needs
 * mf_workspace_size(T, H, D, 1) <= MF_NOALLOC_SCRATCH_BYTES (about 10400 tokens
 * at H*D = 3072); a larger pack returns MF_ERR_UNSUPPORTED and launches nothing.
 * The function allocates nothing. Its first call on a device looks up the array's
 * device address (cudaGetSymbolAddress) with that device current; make that
 * first call before any stream capture. All calls share the array: calls that
 * overlap on the GPU race and must be serialised by the caller. */
#define MF_NOALLOC_SCRATCH_BYTES (64u << 20)
mf_status mf_block_fwd_noalloc(const mf_bf16* x, const mf_bf16* q, const mf_bf16* k,
                               const mf_bf16* v, const float* mod, const int32_t* cu_seqlens_d,
                               const int32_t* cu_seqlens_h, const int32_t* pos_ids,
                               const int32_t* tok_sample, const uint8_t* tok_mod, int32_t S,
                               int32_t H, int32_t D, int32_t rope_axes, float base, float eps,
                               mf_bf16* x_mod, mf_bf16* y, cudaStream_t stream);

/* Packed classifier-free guidance [cfg]: the two branches of an image are two
 * samples of one pack. For each pair (cond, uncond) of sample indices whose
 * samples hold the same number n of image tokens (frames * grid_h * grid_w),
 * output rows [o, o + n) = v_u + w * (v_c - v_u), row i taken from image token
 * i of each sample (a sample's image tokens come first), o = the sum of the
 * earlier pairs' n. The pages name packed CFG but not its combine; this is the
 * usual guidance form. desc: host, S samples (they fix T and the offsets);
 * pairs: host, P >= 1 pairs of distinct samples, P <= MF_MAX_SAMPLES / 2.
 * v: [T][C] bf16; out: [sum n][C] bf16, must not overlap v; C % 8 == 0; w finite.
 * fp32 arithmetic (fma(w, c - u, u)), bf16 round-to-nearest-even output. */
typedef struct {
  int32_t cond;
  int32_t uncond;
} mf_cfg_pair;
mf_status mf_cfg_combine(const mf_bf16* v, const mf_sample_desc* desc, int32_t S,
                         const mf_cfg_pair* pairs, int32_t P, int32_t C, float w, mf_bf16* out,
                         cudaStream_t stream);

/* Modality-specific linear layer [norm]: out[t] = x[t] W[m]^T with m = tok_mod[t]
 * (0 image, 1 text): the image and the text stream of the MMDiT keep their own
 * projection weights. x: [T][K] bf16; W: [2][N][K] bf16 (out features by in
 * features, image weights first); out: [T][N] bf16 (must not overlap x or W).
 * tok_mod: [T] device, from mf_pack_build of the same desc; desc: host, S
 * samples (they fix T and where each modality's rows lie). K % 64 == 0,
 * N % 256 == 0, T <= 131072 (else MF_ERR_UNSUPPORTED). act: MF_ACT_NONE, or
 * MF_ACT_GELU for GELU in its tanh form, 0.5 y (1 + tanh(sqrt(2/pi)(y + 0.044715
 * y^3))), on every output (the MLP's first layer). tcgen05 tensor cores, bf16
 * operands, fp32 accumulation over K and activation, bf16 round-to-nearest-even
 * output. A row whose tok_mod is neither 0 nor 1 is left unwritten. */
#define MF_ACT_NONE 0
#define MF_ACT_GELU 1
mf_status mf_modality_linear(const mf_bf16* x, const mf_bf16* W, const uint8_t* tok_mod,
                             const mf_sample_desc* desc, int32_t S, int32_t K, int32_t N,
                             int32_t act, mf_bf16* out, cudaStream_t stream);

/* One NR-MMDiT block forward around the joint-attention path [norm], [fuse]. The
 * pages give the operations, not the block's wiring; this is the DiT-family block
 * with two gated branches and modality-specific projections (m = tok_mod[t]):
 *   x1 = adaLN(x; mod_attn); q, k, v = x1 W{q,k,v}[m]^T
 *   o  = RoPE + block-diagonal attention (softmax scale 1/sqrt(D)) per sample
 *   y1 = x + gate_attn * (o Wo[m]^T)
 *   x2 = adaLN(y1; mod_mlp); y = y1 + gate_mlp * (GELU(x2 Wup[m]^T) Wdown[m]^T)
 * x, y: [T][hid] bf16 (hid = H * D, a multiple of 256); Wq, Wk, Wv, Wo:
 * [2][hid][hid]; Wup: [2][F][hid]; Wdown: [2][hid][F] (F % 256 == 0; image
 * weights first); mod_attn, mod_mlp: [S][2][3][hid] fp32 (mf_adaln_params);
 * desc, offsets and ids as for mf_block_fwd and mf_modality_linear. Every
 * intermediate is stored in bf16 in the workspace (ws_bytes >=
 * mf_mmdit_workspace_size(T, H, D, F)); the kernels are the library's own
 * (adaLN, linear layers on tcgen05, RoPE, attention, gated residual). y must not
 * overlap x. */
mf_status mf_mmdit_block_fwd(const mf_bf16* x, const mf_bf16* Wq, const mf_bf16* Wk,
                             const mf_bf16* Wv, const mf_bf16* Wo, const mf_bf16* Wup,
                             const mf_bf16* Wdown, const float* mod_attn, const float* mod_mlp,
                             const mf_sample_desc* desc, const int32_t* cu_seqlens_d,
                             const int32_t* cu_seqlens_h, const int32_t* pos_ids,
                             const int32_t* tok_sample, const uint8_t* tok_mod, int32_t S,
                             int32_t H, int32_t D, int32_t F, int32_t rope_axes, float base,
                             float eps, mf_bf16* y, void* workspace, size_t ws_bytes,
                             cudaStream_t stream);
size_t mf_mmdit_workspace_size(int32_t T, int32_t H, int32_t D, int32_t F);

/* Backward of mf_mmdit_block_fwd [norm], [fuse], [train] for the loss gradient dy
 * of y ([T][hid] bf16), with every other argument as in the forward. The
 * forward's intermediates are recomputed into the workspace (bf16, as the
 * forward stores them; z = x2 Wup^T is kept before the GELU), then the chain
 * rule runs through the MLP branch (gate, down projection, GELU, up projection,
 * adaLN) and the attention branch (gate, output projection, attention, RoPE,
 * the three input projections, adaLN), the residual path carrying dy through
 * both. A linear layer's input gradient d_in = d_out W[m] is the tcgen05 linear
 * kernel on the transposed weights; its weight gradient dW[m] = sum over
 * modality-m tokens of d_out^T in is the same kernel on transposes that gather
 * the modality's tokens (a modality without tokens gets dW[m] = 0).
 * Outputs: dx [T][hid] bf16; dWq, dWk, dWv, dWo [2][hid][hid], dWup [2][F][hid],
 * dWdown [2][hid][F] bf16 (image weights first); dmod_attn, dmod_mlp
 * [S][2][3][hid] fp32 (every slot written: shift and scale from the adaLN
 * backward, gate from the gated residual's). Every output is disjoint from every
 * input, from the other outputs and from the workspace (ws_bytes >=
 * mf_mmdit_bwd_workspace_size(T, S, H, D, F)). desc must match the offsets.
 * T and F up to 131072 (else MF_ERR_UNSUPPORTED).
 * bf16 operands and intermediates, fp32 accumulation in every product and sum;
 * the dmod sums use fp32 atomics (their last bits can vary between runs). */
mf_status mf_mmdit_block_bwd(const mf_bf16* dy, const mf_bf16* x, const mf_bf16* Wq,
                             const mf_bf16* Wk, const mf_bf16* Wv, const mf_bf16* Wo,
                             const mf_bf16* Wup, const mf_bf16* Wdown, const float* mod_attn,
                             const float* mod_mlp, const mf_sample_desc* desc,
                             const int32_t* cu_seqlens_d, const int32_t* cu_seqlens_h,
                             const int32_t* pos_ids, const int32_t* tok_sample,
                             const uint8_t* tok_mod, int32_t S, int32_t H, int32_t D, int32_t F,
                             int32_t rope_axes, float base, float eps, mf_bf16* dx, mf_bf16* dWq,
                             mf_bf16* dWk, mf_bf16* dWv, mf_bf16* dWo, mf_bf16* dWup,
                             mf_bf16* dWdown, float* dmod_attn, float* dmod_mlp,
                             void* workspace, size_t ws_bytes, cudaStream_t stream);
size_t mf_mmdit_bwd_workspace_size(int32_t T, int32_t S, int32_t H, int32_t D, int32_t F);

/* Mage-VAE conv block [vae], [vfuse]: the fully convolutional VAE's repeated
 * blocks and their fused normalization - activation - residual chains. The
 * pages give neither the wiring nor the widths; the library takes the diffusion
 * conv nets' residual block
 *   y = x + conv3x3(SiLU(GN(h; gamma2, beta2)); W2, c2),
 *   h = conv3x3(SiLU(GN(x; gamma1, beta1)); W1, c1).
 * Tensors are NHWC bf16 ([N][H][W][C], channels innermost); conv weights
 * [Cout][3][3][Cin] bf16 (tap (dy, dx) reads pixel (h + dy - 1, w + dx - 1),
 * zero outside the image); GroupNorm gamma / beta and conv biases fp32 [C].
 * Supported: C (and Cin, Cout) in {64, 128, 256, 512, 1024, 2048}; C / G a
 * multiple of 8; N * H * W < 2^31; else MF_ERR_UNSUPPORTED.
 *
 * SiLU(GroupNorm(x)) [vfuse]: each sample's channels in G consecutive groups of
 * C / G, normalised over (H, W, C / G) with the population variance and eps,
 * then y = SiLU(xhat * gamma[c] + beta[c]) in one pass over x (statistics by a
 * first pass, merged in a fixed order: repeated calls give the same bits).
 * y must not overlap x. workspace: ws_bytes >= mf_gn_workspace_size(N, H, W, G),
 * disjoint from x and y. */
mf_status mf_group_norm_silu(const mf_bf16* x, const float* gamma, const float* beta, int32_t N,
                             int32_t H, int32_t W, int32_t C, int32_t G, float eps, mf_bf16* y,
                             void* workspace, size_t ws_bytes, cudaStream_t stream);
size_t mf_gn_workspace_size(int32_t N, int32_t H, int32_t W, int32_t G);

/* 3x3 convolution, stride 1, zero padding 1 [vae], as an implicit GEMM on tcgen05
 * tensor cores (bf16 operands, fp32 accumulation): y[n, h, w, o] = sum over taps
 * and input channels of x * Wt, + bias[o] (NULL: none) + residual[n, h, w, o]
 * (NULL: none) added in the epilogue [vfuse], rounded to bf16. x: [N][H][W][Cin];
 * y, residual: [N][H][W][Cout]. y must not overlap x, Wt or bias; residual may
 * equal y (in place) but not overlap it otherwise. */
mf_status mf_conv3x3(const mf_bf16* x, const mf_bf16* Wt, const float* bias,
                     const mf_bf16* residual, int32_t N, int32_t H, int32_t W, int32_t Cin,
                     int32_t Cout, mf_bf16* y, cudaStream_t stream);

/* The whole block: SiLU(GN) -> conv (+ c1) -> SiLU(GN) -> conv (+ c2 + x). Every
 * intermediate is stored in bf16 in the workspace (ws_bytes >=
 * mf_vae_block_workspace_size(N, H, W, C, G)); y must not overlap x, the
 * weights or the workspace. C = Cin = Cout. */
mf_status mf_vae_res_block(const mf_bf16* x, const float* gamma1, const float* beta1,
                           const mf_bf16* W1, const float* c1, const float* gamma2,
                           const float* beta2, const mf_bf16* W2, const float* c2, int32_t N,
                           int32_t H, int32_t W, int32_t C, int32_t G, float eps, mf_bf16* y,
                           void* workspace, size_t ws_bytes, cudaStream_t stream);
size_t mf_vae_block_workspace_size(int32_t N, int32_t H, int32_t W, int32_t C, int32_t G);

/* Bytes of workspace mf_varlen_attn_fwd / mf_block_fwd need (with_rope != 0:
 * room for the fused RoPE's (cos, sin) table, T x D/4 float2, and the rotated
 * k, T x H x D bf16; q is turned inside the attention's load prologue). */
size_t mf_workspace_size(int32_t T, int32_t H, int32_t D, int32_t with_rope);

/* Synchronises `stream`, returns and clears the device error word of the
 * current device (MF_OK if no kernel recorded a failure). */
mf_status mf_get_error(cudaStream_t stream);

/* Limit, in nanoseconds, of every device-side wait of later launches on the
 * current device (default 2e9). A wait that runs out records MF_ERR_TIMEOUT,
 * and the kernel winds down and returns. */
mf_status mf_set_wait_limit_ns(uint64_t ns);

/* Attention kernel of later calls of mf_varlen_attn_fwd, mf_block_fwd and
 * mf_mmdit_block_fwd on the current device, for head_dim 128 (head_dim 64
 * always runs the one-CTA kernel): enable = 0, one CTA per SM, each running
 * two 128-row query tiles; enable = 1, CTA pairs (thread-block clusters of two
 * on two SMs) running each QK^T and PV product as one M = 256 tcgen05 MMA
 * (cta_group::2): each CTA holds its own 128 rows of the two 256-row query tiles,
 * half the keys of every K tile and half the head dims of every V tile, so each
 * SM loads and reads half of the K / V bytes per FLOP. The same products, the
 * same online softmax and epilogue, the same results up to the order of
 * floating-point sums [pack]. Default 0. enable must be 0 or 1. */
mf_status mf_set_attn_cta_pair(int32_t enable);

/* Kernel of later calls of mf_modality_linear (and so of mf_mmdit_block_fwd) on
 * the current device: enable = 0, one CTA per SM, each computing 128-row x
 * 256-column output tiles; enable = 1, CTA pairs (thread-block clusters of two on
 * two SMs) computing 256-row x 256-column tiles as M = 256 tcgen05 MMAs
 * (cta_group::2), each CTA loading its own 128 rows of x and half of each weight
 * tile, so each SM loads a third fewer operand bytes per FLOP. The same products
 * and rounding, the same results up to the order of floating-point sums [norm].
 * Default 1 (measured faster on every pack). enable must be 0 or 1. */
mf_status mf_set_linear_cta_pair(int32_t enable);

/* Kernel of later calls of mf_conv3x3 and mf_vae_res_block on the current device:
 * enable = 0, one CTA per SM, each computing 128-pixel x GN-channel output tiles;
 * enable = 1, CTA pairs (thread-block clusters of two on two SMs) computing two
 * vertically adjacent 128-pixel tiles as M = 256 tcgen05 MMAs (cta_group::2), each
 * CTA loading its own tile's input boxes and half of each weight slice. The same
 * products and rounding, the same results up to the order of floating-point sums
 * [vfuse]. Default 0. enable must be 0 or 1. */
mf_status mf_set_conv_cta_pair(int32_t enable);

/* Instrumentation: while both events are non-NULL, every later call of
 * mf_varlen_attn_fwd / mf_block_fwd on the current device records `start` on its
 * stream right before the attention kernel and `stop` right after it, so the
 * caller can time that kernel alone (cudaEventElapsedTime). (NULL, NULL) turns it
 * off. The events belong to the caller and must outlive the calls that use them. */
mf_status mf_set_attn_timing_events(cudaEvent_t start, cudaEvent_t stop);

/* Self-test of the polynomial 2^x the attention softmax uses for part of its
 * exponentials: y[i] = 2^x[i] for n device floats, evaluated pairwise exactly
 * as in the softmax (x <= 127; inputs below -125 are treated as -125). Relative
 * error <= 7.5e-5 by construction. */
mf_status mf_selftest_exp2_poly(const float* x, float* y, int32_t n, cudaStream_t stream);

/* Self-test of the error channel: launches one CTA that waits on an mbarrier
 * no thread ever arrives at, with a limit of `limit_ns`. The wait runs out, the
 * kernel records MF_ERR_TIMEOUT and returns (no trap, no hang). */
mf_status mf_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MF_H_ */
