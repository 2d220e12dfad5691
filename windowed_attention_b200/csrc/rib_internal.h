// Host-side declarations shared by the translation units of librib.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>
#include <string>

#include "../../include/rib.h"

namespace rib {

// thread-local message for rib_last_error()
void set_error(const std::string& msg);
rib_status fail(rib_status s, const std::string& msg);
rib_status cuda_fail(cudaError_t e, const char* what);

// Device address of the error word that bounded waits write (current device).
int* device_error_word();

// Device address of a __device__ symbol of this library on the current
// device, looked up once per (slot, device) with that device current and
// cached; err receives the lookup's status.
enum { kSymErrorWord = 0, kSymGateScratch = 1, kSymSlots = 2 };
void* cached_symbol_address(int slot, const void* symbol, cudaError_t* err);

// The CLA gate's argument checks (every entry point of the gate) and its
// two-pass form (depthwise into D, then the pointwise token GEMM).
rib_status check_gate_args(const char* who, const void* X, rib_dtype xdtype, int B, int H, int W, int C,
                           const float* Wdw, const float* bdw, const void* Wpw, const float* bpw, const void* sig_gate);
rib_status cla_gate_two_pass(const char* who, const void* X, int B, int H, int W, int C, const float* Wdw,
                             const float* bdw, const void* Wpw, const float* bpw, void* sig_gate, void* D,
                             cudaStream_t stream);

// Number of SMs of the current device.
int sm_count();

// cuTensorMapEncodeTiled through the runtime's driver entry point.
CUresult encode_tiled(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t rank, void* addr,
                      const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                      CUtensorMapSwizzle swizzle);

// Window tiling of one M x M window into 128-token rectangles (rows x cols).
struct WindowTiling {
  int tc, tr;   // columns x rows of one 128-token tile
};
bool window_tiling(int M, WindowTiling* t);

// Kernel launchers (return cudaGetLastError() of the launch).
struct AttnLaunch {
  int B, H, W, C, heads, dh, DP, M, tc, tr;
  int mask_padding;   // exclude padded keys from the softmax
  int out_f32;        // Y and the residual are fp32
  int out_f16;        // Y and the residual are fp16 (neither: bf16)
  float scale_log2;
  const void *Qc, *Kc, *V, *qp, *kp, *gate, *resid;
  void* Y;
  float* lse;
  void* O_out;
};
cudaError_t launch_window_attention(const AttnLaunch& a, cudaStream_t stream);

struct AttnBwdLaunch {
  int B, H, W, C, heads, dh, DP, M, tc, tr;
  float scale;
  const void *Qc, *Kc, *V, *qp, *kp, *dO;
  const float* lse;
  float *dQc, *dKc, *dV, *dQp, *dKp;
  float *ws_q, *ws_k;   // per-window partials of dQp, dKp
  void *qf, *qpf;       // (dh + 2 <= DP) the folded Q'' content and rank tensors
};
cudaError_t launch_window_attention_bwd(const AttnBwdLaunch& a, cudaStream_t stream);
cudaError_t launch_bwd_prep(const void* dY, const void* gate, const void* O, void* dO, float* Dsum, void* dG, int B,
                            int H, int W, int C, int heads, int M, float scale, cudaStream_t stream);
// token chunks of the coordinate-MLP weight-gradient reduction (fixed, so
// the summation order, and the result, are deterministic)
constexpr int kPosBwdChunks = 64;
cudaError_t launch_pos_encode_bwd(const rib_mlp_desc& m, int M, const float* dqp, const float* dkp, float* dWh,
                                  float* dbh, float* dWpq, float* dWpk, float* ws, cudaStream_t stream);

struct GemmJob {
  const void* Wt;     // bf16 [K][w_cols]
  void* out;          // mode 0: [rows][N] bf16 or fp16; mode 1: bf16 [rows][n_real]
  int N;              // MMA N of this job (multiple of 16, <= 256)
  int DP;             // mode 0: padded per-head width of this job's output
  int out_f16;        // 1 -> fp16 output (saturating at +-65504), 0 -> bf16
  int ones_col;       // mode 0: >= 0 -> columns head*DP + d, d >= ones_col, are written as 1
  float scale;        // mode 0: multiplier of the product
  const float* bias;  // mode 1: fp32 [n_real] or null
};
struct GemmLaunch {
  const void* A;      // bf16 [B][H][W][K]
  int B, H, W;        // image of the A rows
  int Hp, Wp;         // mode 0: output image padded to these (rows outside H x W read as 0)
  int K;              // reduction size = channels (multiple of 4, <= 256)
  int a_f16;          // A (the map) is fp16: the product runs in fp16 (weights converted)
  int mode;           // 0: head-padded projection, 1: pointwise + bias + sigmoid
  int heads, dh;      // projection column map: n = head*DP + d <- weight column head*dh + d
  int n_real;         // mode 1: stored columns (= C)
  int n_valid;        // mode 1: columns with weights and bias (0: all n_real)
  int gelu;           // mode 1: GELU (erf form) instead of the sigmoid
  int w_cols;         // columns of each Wt
  int njobs;
  GemmJob jobs[3];
};
cudaError_t launch_token_gemm(const GemmLaunch& g, cudaStream_t stream);

// Projection backward: dX = sum_j (s_j g_j) W_j^T (written), dW_j = X^T (s_j g_j)
// (written); g_j fp32 [B][Hp][Wp][heads][32], W_j and X bf16.
struct QkvBwdLaunch {
  int B, H, W, Hp, Wp, C, heads;
  const float* g[3];
  float s[3];
  const void* Wt[3];
  const void* X;
  float* dX;
  float* dW[3];
};
cudaError_t launch_qkv_project_bwd(const QkvBwdLaunch& a, void* ws, cudaStream_t stream);
// Gate backward: dD = dG Wpw^T (into dD), dX += DWConv3x3^T(dD), dWpw, dWdw,
// dbdw, dbpw (written).
struct GateBwdLaunch {
  int B, H, W, C;
  const void* X;
  const float* Wdw;
  const void* Wpw;
  const void* D;
  const void* dG;
  float* dD;
  float* dX;
  float *dWdw, *dbdw, *dWpw, *dbpw;
};
cudaError_t launch_cla_gate_bwd(const GateBwdLaunch& a, void* ws, cudaStream_t stream);

// Weight-gradient reductions write one [C][C] partial sum per chunk of
// tokens (and job); the sums add them in chunk order (no atomics), so the
// gradients are bit-identical from run to run.
constexpr int kWgradChunks = 144;
inline size_t align256(size_t v) { return (v + 255) / 256 * 256; }
size_t wgrad_partial_bytes(int C);
cudaError_t launch_wgrad_partial_sum(const float* partial, int chunks, int jobs, int n, float* o0, float* o1,
                                     float* o2, cudaStream_t stream);
// Tensor-core forms (layer_bwd_tc.cu): maps with W*C % 8 == 0, 16-byte
// aligned, C in [32, 256], W >= 32, H >= 4.
bool tc_bwd_supported(const void* map, int H, int W, int C);
size_t tc_bwd_weight_image_bytes(int C, int heads, bool projection);
cudaError_t launch_qkv_project_bwd_tc(const QkvBwdLaunch& a, void* ws, cudaStream_t stream);
cudaError_t launch_gate_bwd_tc_gemms(const GateBwdLaunch& a, uint8_t* img, float* partial, cudaStream_t stream,
                                     int* chunks_out);
size_t qkv_project_bwd_ws_bytes(int B, int H, int W, int C, int heads);
size_t gate_bwd_ws_bytes(int B, int H, int W, int C);

// Fused CLA gate (depthwise 3x3 into the pointwise tcgen05 GEMM's operand,
// sigmoid epilogue); D_out (optional) receives the depthwise output.
bool cla_gate_fused_supported(const void* X, int B, int H, int W, int C);
// The same kernel in general: depthwise 3x3 over Cin channels (weights on the
// first Cw), pointwise to Cout; ffn = 1: ConvFFN epilogue (h + DWConv(h), then
// xres += . W + b in fp32), ffn = 0: gate epilogue (sigmoid, bf16 out).
bool dw_pw_fused_supported(const void* X, int W, int Cin, int Cout);
cudaError_t launch_dw_pw_fused(const void* X, int B, int H, int W, int Cin, int Cw, int Cout, const float* Wdw,
                               const float* bdw, const void* Wpw, const float* bpw, void* out, void* D_out, float* xres,
                               int ffn, int x_f16, cudaStream_t stream);
// (ffn = 1 runs the pointwise product in fp16; x_f16 = 1 reads X as fp16)
cudaError_t launch_cla_gate_fused(const void* X, int x_f16, const float* Wdw, const float* bdw, const void* Wpw,
                                  const float* bpw, void* out, void* D_out, int B, int H, int W, int C, cudaStream_t stream);
cudaError_t launch_dwconv3x3(const void* X, const float* Wdw, const float* bdw, void* out, int B, int H, int W,
                             int C, cudaStream_t stream);
// xtype: 0 bf16, 1 fp32, 2 fp16 input
cudaError_t launch_layernorm(const void* x, int xtype, void* y, int y_f16, long long T, int C, const float* gamma,
                             const float* beta, float eps, cudaStream_t stream);
cudaError_t launch_f32_to_bf16(const float* x, void* y, size_t n, cudaStream_t stream);
cudaError_t launch_bf16_to_f32(const void* x, float* y, size_t n, cudaStream_t stream);
cudaError_t launch_pos_encode(const rib_mlp_desc& m, int M, void* qp, void* kp, cudaStream_t stream);

}  // namespace rib
