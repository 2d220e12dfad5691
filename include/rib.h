/*
 * librib - windowed RIB attention with CLA gate on B200 (sm_100a).
 *
 * The operation (RIB/SST write-up, "FlashAttention-accelerated
 * super-resolution Transformer", omica.com.cn, sections 2.2 and 2.3):
 * per non-overlapping M x M window and head,
 *     S = Qc Kc^T / sqrt(D) + Qp Kp^T / sqrt(R)      (one product of the
 *         concatenations [Qc/sqrt(D), Qp/sqrt(R)] and [Kc, Kp])
 *     O = softmax(S) V * sigmoid(PWConv(DWConv3x3(X)))
 * where Qp, Kp come from a coordinate MLP over Fourier features of the
 * window grid (section 2.2 CoordinateEncoder / implicit neural field) and
 * are computed once per window size (section 5.2, position cache).
 *
 * Conventions shared by every entry point:
 *  - All pointers are DEVICE pointers unless a comment says otherwise. The
 *    caller owns every buffer; the library never allocates device memory.
 *  - Feature maps are channels-last [B][H][W][C] (the write-up's b (h w) c).
 *  - bf16 is IEEE-style bfloat16 stored as 16-bit words.
 *  - Weights use the "x @ W" orientation: W[in][out], row-major.
 *  - Calls are ordered on the given cudaStream_t (0 = legacy default
 *    stream) and never synchronise. Arguments are validated on the host
 *    before anything is launched; a failed check launches nothing.
 *  - Every pointer is aligned at least to its element size (2 bytes for
 *    bf16/fp16 data, 4 for fp32); a call that needs more states it. A
 *    pointer that misses its alignment gives RIB_ERR_ALIGNMENT.
 *  - Every call returns rib_status; rib_last_error() then holds a message
 *    (thread-local, valid until the next call on the same thread).
 *  - Kernels never wait without a bound. A wait that runs out records a
 *    site code on the device; rib_device_error() reads and clears it.
 */
#ifndef RIB_H_
#define RIB_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#pragma GCC visibility push(default)
#endif
#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RIB_OK = 0,
  RIB_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, inconsistent shapes */
  RIB_ERR_UNSUPPORTED = 2,   /* shape outside what the kernels implement (see each call) */
  RIB_ERR_ALIGNMENT = 3,     /* a pointer misses the alignment a call requires */
  RIB_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed (message has the code) */
  RIB_ERR_TIMEOUT = 5        /* a device-side bounded wait ran out (from rib_device_error) */
} rib_status;

/* Storage types of maps at the boundary. RIB_F16 is the fp16 path of the
 * write-up's FP16 mixed-precision training (section 3.3): fp16 maps into the
 * projections, the gate and LayerNorm, fp16 Y out of the attention store; the
 * tensor-core operands inside stay bf16 (the projection runs in fp16 against
 * fp16 copies of its bf16 weights). The backward entry points take bf16. */
typedef enum { RIB_BF16 = 0, RIB_F32 = 1, RIB_F16 = 2 } rib_dtype;

/* Message of the last failed call on this thread ("" if none). Host pointer,
 * owned by the library. */
const char* rib_last_error(void);

/* Library version: major*10000 + minor*100 + patch. */
int rib_version(void);

/* Synchronises `stream`, then reads and clears the device-side error word
 * that bounded waits write. Returns RIB_OK, RIB_ERR_TIMEOUT (message names
 * the wait site) or RIB_ERR_CUDA (a sticky CUDA error, e.g. a fault). */
rib_status rib_device_error(cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Coordinate MLP weights of one layer (section 2.2, implicit neural field):
 *   r  = [c, sin(2^0 c), cos(2^0 c), ..., sin(2^(L-1) c), cos(2^(L-1) c)]
 *        (2+4L values per token, c = (y, x) on linspace(-1,1,M)^2)
 *   h  = ReLU(r Wh + bh)          Wh [2+4L][hidden], bh [hidden]
 *   Qp = h Wpq, Kp = h Wpk        Wpq, Wpk [hidden][heads*R], head-major
 * All four are fp32 device pointers.
 * ---------------------------------------------------------------------- */
typedef struct {
  int L;          /* Fourier bands, 1..16 */
  int hidden;     /* MLP hidden width, 1..256 */
  int heads;      /* attention heads, 1..16 */
  int R;          /* rank of the positional features; must be 16 */
  const float* Wh;
  const float* bh;
  const float* Wpq;
  const float* Wpk;
} rib_mlp_desc;

/* Bytes of one Qp (or Kp) cache for window side `window`:
 * heads * window * window * R * 2. */
size_t rib_pos_cache_bytes(const rib_mlp_desc* mlp, int window);

/* a1+a2: position features of an M x M window (section 2.2; cached once per
 * window size as in section 5.2). Writes
 *   qp_cache[h][i][j][r] = bf16( Qp[h, i*M+j, r] / sqrt(R) )
 *   kp_cache[h][i][j][r] = bf16( Kp[h, i*M+j, r] )
 * i.e. the 1/sqrt(R) of the score is folded into the cached Qp.
 * cache_bytes is the size of EACH buffer (>= rib_pos_cache_bytes).
 * Buffers 16-byte aligned. window 1..256, L 1..16, hidden 1..256, heads
 * 1..16. The Fourier features are evaluated in double precision (their
 * arguments reach 2^(L-1) rad), the MLP in fp32. */
rib_status rib_pos_encode(const rib_mlp_desc* mlp, int window, void* qp_cache, void* kp_cache,
                          size_t cache_bytes, cudaStream_t stream);

/* Padded per-head width used by the content tensors: dh rounded up to 16. */
int rib_head_pad(int C, int heads);

/* a3: content projections (the write-up takes Qc, Kc, V as given pixel
 * content features; they are X Wq, X Wk, X Wv, bias-free), written in the
 * window-padded, head-major layout the attention kernel reads:
 *   X      [B][H][W][C] bf16 (convert fp32 maps with rib_f32_to_bf16)
 *   Wq,Wk,Wv bf16 [C][C]  (in, out)
 *   window the window side M; the outputs cover the map zero-padded at the
 *          bottom/right to Hp = ceil(H/M)*M rows and Wp = ceil(W/M)*M columns
 *   Qc, Kc bf16 [B][Hp][Wp][heads][DP], DP = rib_head_pad(C, heads): entry
 *          d < dh holds channel head*dh+d (Qc multiplied by q_scale; pass
 *          1/sqrt(dh) for the write-up's Qc/sqrt(D)); Qc's entries d >= dh
 *          are 0 and Kc's are 1 (every token; when dh < DP): the attention
 *          kernels carry per-row constants of the softmax through them, and
 *          since Qc's entries there are 0 the score is unchanged
 *   V      bf16 [B][Hp][Wp][heads][32]: entry d < dh holds channel
 *          head*dh+d, entries d >= dh are 1 (every token, padding included:
 *          the attention kernel sums the softmax denominator through them)
 * Padded tokens (outside H x W) have Qc = Kc = 0 and V = 0 apart from the
 * ones columns.
 * X may be fp16 (xdtype RIB_F16): the product then runs in fp16 with the
 * weights converted to fp16; the outputs stay as above.
 * Requirements: C % heads == 0, dh = C/heads even and <= 30, heads <= 8,
 * C <= 256, C % 4 == 0, X 8-byte aligned, outputs 16-byte aligned. */
rib_status rib_qkv_project(const void* X, rib_dtype xdtype, int B, int H, int W, int C, int heads, int window,
                           const void* Wq, const void* Wk, const void* Wv, float q_scale,
                           void* Qc, void* Kc, void* V, cudaStream_t stream);

/* a5+a6: CLA gate (section 2.3): sig_gate = sigmoid(PWConv(DWConv3x3(X))).
 *   X        [B][H][W][C] bf16, or fp16 with xdtype RIB_F16 (fp16 maps need
 *            W*C % 8 == 0; xdtype RIB_F32 is refused with
 *            RIB_ERR_UNSUPPORTED: convert fp32 maps with rib_f32_to_bf16)
 *   Wdw      fp32 [C][3][3], bdw fp32 [C]   (zero padding 1 at the border)
 *   Wpw      bf16 [C][C] (in, out), bpw fp32 [C]
 *   sig_gate bf16 [B][H][W][C]
 *   workspace >= cla_gate_workspace_size(): holds DWConv3x3(X) in bf16.
 * Requirements: C % 4 == 0, C <= 256, X/sig_gate/workspace 16-byte aligned. */
size_t cla_gate_workspace_size(int B, int H, int W, int C);
rib_status cla_gate(const void* X, rib_dtype xdtype, int B, int H, int W, int C,
                    const float* Wdw, const float* bdw, const void* Wpw, const float* bpw,
                    void* sig_gate, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* cla_gate without a workspace, for callers that cannot allocate device
 * memory: hosts that forbid allocation after start-up (deployment runtimes
 * with a fixed memory plan, plugin interfaces that hand the library only its
 * inputs and outputs). The paper has no counterpart of this; it is an
 * interface for such callers, computing exactly what cla_gate computes.
 *
 * The depthwise intermediate lives in a fixed array of this library,
 * RIB_GATE_STATIC_SCRATCH_BYTES (16 MiB) on every device that loads the
 * library, held until the process exits. Arguments as for cla_gate minus the
 * workspace. Calls with B*H*W*C*2 > RIB_GATE_STATIC_SCRATCH_BYTES are
 * rejected (RIB_ERR_UNSUPPORTED) before anything is launched; use cla_gate
 * for them. The call allocates nothing.
 *  - The first call on each device looks up the array's address on that
 *    device (with that device current); make that first call before any
 *    stream capture.
 *  - Every call on a device uses the same array and leaves its contents
 *    behind; nothing in it needs clearing, since each call writes every
 *    element it later reads. Calls whose executions overlap on the GPU
 *    (different streams, no ordering between them) race on the array:
 *    order them. */
#define RIB_GATE_STATIC_SCRATCH_BYTES (16u << 20)
rib_status cla_gate_static_scratch(const void* X, rib_dtype xdtype, int B, int H, int W, int C,
                                   const float* Wdw, const float* bdw, const void* Wpw, const float* bpw,
                                   void* sig_gate, cudaStream_t stream);

/* ConvFFN of the full SST block (section 3.1 "模型架构设计": each block is
 * LayerNorm -> RIB attention -> CLA -> ConvFFN with FFN expansion 1.25; the
 * write-up names the ConvFFN without defining it, and this is the reading the
 * library takes): with xn = LayerNorm(x),
 *   h  = GELU(xn W1 + b1)                 (erf form; hidden = 1.25 C)
 *   x += (h + DWConv3x3(h)) W2 + b2       (zero padding 1, per-channel filter and bias)
 *   xn  [B][H][W][C] of dtype xndtype (RIB_BF16 or RIB_F16; 8-byte
 *       aligned); with fp16 the first map's product runs on fp16 operands
 *       (W1 converted, exact in fp16's range)
 *   x   fp32 [B][H][W][C], updated in place (the block's residual stream;
 *       16-byte aligned)
 *   W1  bf16 [C][hidden], b1 fp32 [hidden], Wf fp32 [hidden][3][3],
 *   bf  fp32 [hidden], W2 bf16 [hidden][C], b2 fp32 [C]
 *   workspace >= rib_conv_ffn_workspace_size(): h, fp16 [B][H][W][hidden
 *       rounded up to 8], 16-byte aligned.
 * Two kernels: the first linear map on the tensor cores with bias and GELU in
 * its epilogue, then one pass that computes h + DWConv3x3(h) straight into the
 * second map's tensor-core operand and adds the result into x. h, that
 * operand and W2 are held in fp16 (saturating conversions): xn is a
 * LayerNorm output, so h is bounded, and fp16's finer steps keep the two
 * roundings between the linear maps small.
 * Requirements: C % 4 == 0, C <= 256, hidden <= 256 (hidden widths above
 * 256 return RIB_ERR_UNSUPPORTED; a shape whose tiles do not fit in shared
 * memory would too, which no shape within these limits does for the first
 * map). */
size_t rib_conv_ffn_workspace_size(int B, int H, int W, int hidden);
rib_status rib_conv_ffn(const void* xn, rib_dtype xndtype, float* x, int B, int H, int W, int C, int hidden,
                        const void* W1, const float* b1, const float* Wf, const float* bf, const void* W2,
                        const float* b2, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* a4: fused windowed RIB attention (sections 2.2-2.3). */
typedef struct {
  int B, H, W;        /* image; windows tile the map zero-padded bottom/right */
  int C, heads;       /* dh = C/heads (even, <= 30), DP = rib_head_pad(C, heads) */
  int R;              /* must be 16 */
  int window;         /* M: any multiple of 16 from 16 to 256 (a 128-query
                         tile is a tc x tr rectangle of the window, tc the
                         largest power of two <= 128 dividing M); the GPU
                         parity tests cover 16, 32, 64 and 96 */
  float softmax_scale;/* extra logit multiplier; 1.0 when Qc carries
                         1/sqrt(dh) and qp_cache carries 1/sqrt(R) */
  int mask_padding;   /* 0: padded pixels are keys with Kc = V = 0 (the
                         default reading of the zero padding); 1: they are
                         excluded from every row's softmax (key-padding mask).
                         Forward only: the backward entry points reject 1. */
  rib_dtype out_dtype;/* storage of Y and the residual: RIB_BF16 (0),
                         RIB_F32 (an fp32 residual stream, e.g. a block stack
                         x <- x + Y(LN(x))) or RIB_F16 (the fp16 path; values
                         saturate at +-65504); the backward ignores it */
} rib_attn_desc;

/* Per (window, head): S = Qc Kc^T + Qp Kp^T (two accumulating tensor-core
 * products, no S in memory), P = softmax(softmax_scale * S), O = P V, then
 *   Y[b][y][x][head*dh + d] = O[d] * sig_gate[...] (+ residual[...])
 * for every real pixel (window reverse + crop fused in the store).
 *   Qc, Kc, V  rib_qkv_project's window-padded layout for this window
 *              (Qc, Kc bf16 [B][Hp][Wp][heads][DP], V bf16 [B][Hp][Wp][heads][32]
 *              with its ones columns at d >= dh, and Kc's at d >= dh when
 *              dh < DP: the kernel relies on both)
 *   qp_cache, kp_cache  bf16 [heads][M][M][R] (rib_pos_encode's layout)
 *   sig_gate   bf16 [B][H][W][C] or NULL (no gate: factor 1)
 *   residual   [B][H][W][C] in desc->out_dtype, or NULL; may alias Y
 *   Y          [B][H][W][C] in desc->out_dtype (bf16 or fp32)
 *   lse        fp32 [B][heads][Hp][Wp] natural-log row log-sum-exp of the
 *              scaled logits, or NULL (needed by the backward)
 *   O_out      bf16 [B][H][W][heads][DP] ungated attention output or NULL
 *              (needed by the backward)
 * Padded pixels are keys with Kc = V = 0 and their grid Kp (they enter the
 * softmax denominator) unless desc->mask_padding is 1 (then every row's
 * softmax skips them); their query rows are computed and dropped. All
 * tensors 16-byte aligned. */
/* Workspace of rib_window_attention in bytes: always 0, since the fused
 * kernel keeps S, P and the running softmax state on chip (TMEM, registers)
 * and writes only Y, lse and O_out. Provided so that callers size every
 * call's workspace the same way. */
size_t rib_window_attention_workspace_size(const rib_attn_desc* desc);
rib_status rib_window_attention(const rib_attn_desc* desc, const void* Qc, const void* Kc, const void* V,
                                const void* qp_cache, const void* kp_cache, const void* sig_gate,
                                const void* residual, void* Y, float* lse, void* O_out,
                                cudaStream_t stream);

/* a8: backward of the windowed RIB attention and of the CLA gate's product
 * (training). With S = Qc Kc^T + Qp Kp^T as in rib_window_attention, P its
 * softmax and O = P V, the gradients from dO are (RIB/SST write-up section
 * 2.2: the concatenated product splits at the content/position boundary)
 *   D = rowsum(dO * O),  dS = softmax_scale * P * (dO V^T - D),
 *   dQc = dS Kc, dQp = dS Kp, dKc = dS^T Qc, dKp = dS^T Qp, dV = P^T dO,
 * all with respect to the tensors as rib_qkv_project / rib_pos_encode store
 * them (Qc including its q_scale, the cached Qp including 1/sqrt(R)).
 *
 * Step 1, rib_attention_bwd_prep: from the upstream gradient dY of
 * Y = O * sig_gate, with s = desc->softmax_scale,
 *   dO   bf16 [B][Hp][Wp][heads][32] in the padded layout: columns d < dh
 *        hold s * dY * sig_gate; columns dh and dh+1 hold -s*D as a pair of
 *        bf16 values (hi, lo) whose sum is -s*D, the rest 0 (all 0 in the
 *        padding). V's columns d >= dh are 1, so the backward's product
 *        dO V^T is s * (dO V^T - D) directly.
 *   Dsum fp32 [B][heads][Hp][Wp]     = D = rowsum(dY * sig_gate * O) (from
 *        the stored bf16 values; informational, the backward reads dO)
 *   dG   bf16 [B][H][W][C] or NULL   = dY * O * sig_gate * (1 - sig_gate)
 *        (gradient of the gate's pre-activation G)
 * with dY, sig_gate bf16 [B][H][W][C] and O the forward's O_out
 * (bf16 [B][H][W][heads][DP]). dY, sig_gate, dG and Dsum 4-byte aligned,
 * O and dO 16-byte aligned (the kernel moves eight columns at a time). */
rib_status rib_attention_bwd_prep(const rib_attn_desc* desc, const void* dY, const void* sig_gate, const void* O,
                                  void* dO, float* Dsum, void* dG, cudaStream_t stream);

/* Step 2, rib_window_attention_bwd: P is recomputed from the forward's lse.
 *   Qc, Kc, V, qp_cache, kp_cache  the forward's inputs
 *   lse   fp32 [B][heads][Hp][Wp] from the forward
 *   dO    from rib_attention_bwd_prep (Dsum is not read; it may be any
 *         16-byte-aligned pointer, or rib_attention_bwd_prep's Dsum)
 *   dQc, dKc, dV  fp32 [B][Hp][Wp][heads][32] (columns >= dh carry no
 *         gradient of the layer: ignore them)
 *   dQp, dKp      fp32 [heads][M][M][16]: summed over every window and image
 *         (the gradient of the two position caches)
 *   workspace >= rib_window_attention_bwd_workspace_size(desc): per-window
 *         partials of dQp/dKp, summed in a fixed order (deterministic), and,
 *         for padded heads with two spare columns (dh + 2 <= DP), the folded
 *         query operands: bf16(l2 * Qc) with -log2(e) * lse in columns dh,
 *         dh+1 and bf16(l2 * Qp) per token (l2 = softmax_scale * log2(e)),
 *         so that the score product itself yields log2 of P.
 * All tensors 16-byte aligned. */
size_t rib_window_attention_bwd_workspace_size(const rib_attn_desc* desc);
rib_status rib_window_attention_bwd(const rib_attn_desc* desc, const void* Qc, const void* Kc, const void* V,
                                    const void* qp_cache, const void* kp_cache, const float* lse, const void* dO,
                                    const float* Dsum, float* dQc, float* dKc, float* dV, float* dQp, float* dKp,
                                    void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Step 3, rib_pos_encode_bwd: gradients of the coordinate-MLP weights (section
 * 2.2 implicit neural field) from the gradients of the two caches of window
 * side `window` (dqp_cache, dkp_cache: fp32 [heads][M][M][16] as returned
 * above). Outputs fp32 dWh [2+4L][hidden], dbh [hidden], dWpq, dWpk
 * [hidden][heads*R]; the features and hidden activations are recomputed.
 * workspace >= rib_pos_encode_bwd_workspace_size(). Deterministic. */
size_t rib_pos_encode_bwd_workspace_size(const rib_mlp_desc* mlp, int window);
rib_status rib_pos_encode_bwd(const rib_mlp_desc* mlp, int window, const float* dqp_cache, const float* dkp_cache,
                              float* dWh, float* dbh, float* dWpq, float* dWpk, void* workspace,
                              size_t workspace_bytes, cudaStream_t stream);

/* Step 4, rib_qkv_project_bwd: backward of the content projections (the
 * content features Qc = X Wq, Kc = X Wk, V = X Wv). From the gradients of the
 * stored projections (rib_window_attention_bwd's dQc, dKc, dV: fp32
 * [B][Hp][Wp][heads][32] for this window's padding; dQc is taken as the
 * gradient of the stored Qc = q_scale * X Wq, so pass the forward's q_scale;
 * columns >= dh are ignored), with g_q = q_scale * dQc, g_k = dKc, g_v = dV
 * restricted to real pixels:
 *   dX  = g_q Wq^T + g_k Wk^T + g_v Wv^T   fp32 [B][H][W][C], overwritten
 *   dWq = X^T g_q, dWk = X^T g_k, dWv = X^T g_v   fp32 [C][C], overwritten
 * X bf16 [B][H][W][C] (8-byte aligned), Wq/Wk/Wv bf16 [C][C] as in the
 * forward. workspace >= rib_qkv_project_bwd_workspace_size() bytes, 16-byte
 * aligned (weights re-laid for the tensor cores and per-chunk partial sums of
 * the weight gradients). Maps with W*C % 8 == 0, a 16-byte aligned X, C >= 32,
 * W >= 32 and H >= 4 run on the tensor cores, the fp32 gradients entering the
 * products as bf16 hi + lo pairs (about 2^-17 relative); other maps on fp32
 * CUDA cores. The weight gradients are sums of per-chunk partials added in a
 * fixed order: bit-identical from run to run on the same GPU. Same shape
 * limits as rib_qkv_project. */
size_t rib_qkv_project_bwd_workspace_size(int B, int H, int W, int C, int heads);
rib_status rib_qkv_project_bwd(const void* X, rib_dtype xdtype, int B, int H, int W, int C, int heads, int window,
                               const void* Wq, const void* Wk, const void* Wv, float q_scale, const float* dQc,
                               const float* dKc, const float* dV, float* dX, float* dWq, float* dWk, float* dWv,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Step 5, cla_gate_bwd: backward of the CLA gate sigma(PWConv(DWConv3x3(X)))
 * (section 2.3) from dG, the gradient of its pre-activation G = D Wpw + bpw
 * (rib_attention_bwd_prep's dG, bf16 [B][H][W][C]):
 *   dD   = dG Wpw^T                       (fp32, kept in the workspace)
 *   dX  += DWConv3x3^T(dD)                fp32 [B][H][W][C], ADDED to dX (call
 *          after rib_qkv_project_bwd, which writes dX)
 *   dWpw = D^T dG [C][C], dbpw = sum dG [C],
 *   dWdw[c][ky][kx] = sum_p X[p + (ky-1, kx-1)][c] dD[p][c] [C][3][3],
 *   dbdw = sum dD [C]                     fp32, overwritten
 * X bf16 [B][H][W][C]; D = the depthwise output the forward left in
 * cla_gate's workspace (bf16 [B][H][W][C]); Wdw fp32 [C][3][3], Wpw bf16
 * [C][C]. workspace >= cla_gate_bwd_workspace_size() bytes (dD, the
 * pointwise weights re-laid for the tensor cores, per-chunk partial sums).
 * dD and dWpw run on the tensor cores for maps with W*C % 8 == 0, C >= 32,
 * W >= 32 and H >= 4 (else on fp32 CUDA cores); every reduction over pixels
 * adds per-chunk partials in a fixed order, so the results are bit-identical
 * from run to run on the same GPU. C % 4 == 0, C <= 256; X, D, dG, dX and the
 * workspace 16-byte aligned. */
size_t cla_gate_bwd_workspace_size(int B, int H, int W, int C);
rib_status cla_gate_bwd(const void* X, rib_dtype xdtype, int B, int H, int W, int C, const float* Wdw, const void* Wpw,
                        const void* D, const void* dG, float* dX, float* dWdw, float* dbdw, float* dWpw, float* dbpw,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Diagnostic (the pages have no counterpart): launches one warp that waits
 * on a barrier nothing arrives on, with a bounded wait of limit_us
 * microseconds (1..1000000) instead of the kernels' 1 s. The wait runs out,
 * records its site (901) in the device error word and returns, so the next
 * rib_device_error() on the stream reports RIB_ERR_TIMEOUT (and clears the
 * word) while the context stays usable: the failure path of every bounded
 * wait, exercised without faulting or hanging the GPU. */
rib_status rib_selftest_wait_timeout(int limit_us, cudaStream_t stream);

/* Diagnostic (the pages have no counterpart): the issue rate of tcgen05.mma,
 * which bounds the attention kernels because their products are narrow
 * (N = 16 to 64: the head and rank widths). Launches ctas_per_sm (1..4) CTAs
 * per SM, their shared memory sized so that no more share an SM, each with
 * issuers_per_cta (1..4) threads in separate warps; every thread issues a
 * chain of `mmas` (1..65536) kind::f16 products of M = 128, K = 16 and
 * width n (a multiple of 16, 16..256) from zero-filled shared-memory
 * operands into its own TMEM accumulator (issuers_per_cta * n <= 512 /
 * ctas_per_sm rounded down to a power of two). cycles: DEVICE buffer of
 * sm_count * ctas_per_sm * issuers_per_cta * 2 unsigned 64-bit values,
 * entry ((cta * issuers_per_cta + i) * 2 + {0, 1}) = clock64 cycles of
 * thread i of that CTA from its first issue to its last issue, and to the
 * completion of its chain (0 if its bounded wait ran out: the device error
 * word then holds site 902). spans: DEVICE buffer of sm_count * ctas_per_sm
 * * 3 values or null; entry (cta * 3 + {0, 1, 2}) = the CTA's SM id and the
 * globaltimer (ns) before its threads' first issue and after their chains
 * completed, which shows whether the CTAs of an SM ran at the same time.
 * Errors: RIB_ERR_INVALID_ARG for an argument out of range or a null cycles
 * buffer; launch failures as RIB_ERR_CUDA. Asynchronous on `stream`. */
rib_status rib_selftest_mma_rate(int ctas_per_sm, int issuers_per_cta, int n, int mmas, unsigned long long* cycles,
                                 unsigned long long* spans, cudaStream_t stream);

/* a7: LayerNorm over C per token (section 3.1 block: LayerNorm -> RIB
 * attention -> CLA). y = (x - mean) / sqrt(var + eps) * gamma + beta, biased
 * variance, fp32 statistics. x dtype xdtype (bf16, fp32 or fp16), y dtype
 * ydtype (RIB_BF16, or RIB_F16 with a saturating conversion: the normalised
 * values are small, and fp16's 11-bit significand keeps the rounding of a
 * block's input 8 times smaller than bf16's), gamma/beta fp32 [C] or NULL (1
 * and 0). T = number of tokens. C <= 1024, C % 4 == 0, eps > 0; x 8-byte
 * aligned (16 for fp32), y 8-byte aligned. */
rib_status rib_layernorm(const void* x, rib_dtype xdtype, void* y, rib_dtype ydtype, int T, int C,
                         const float* gamma, const float* beta, float eps, cudaStream_t stream);

/* Elementwise fp32 -> bf16 rounding (round to nearest even) of n values;
 * used to bring fp32 feature maps to the bf16 operand type. x 16-byte and
 * y 8-byte aligned; n == 0 launches nothing. */
rib_status rib_f32_to_bf16(const float* x, void* y, size_t n, cudaStream_t stream);

/* Elementwise bf16 -> fp32 widening (exact) of n values; used to start an
 * fp32 residual stream (rib_attn_desc.out_dtype = RIB_F32) from a bf16 map.
 * x 8-byte and y 16-byte aligned; n == 0 launches nothing. */
rib_status rib_bf16_to_f32(const void* x, float* y, size_t n, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#if defined(__GNUC__)
#pragma GCC visibility pop
#endif
#endif /* RIB_H_ */
