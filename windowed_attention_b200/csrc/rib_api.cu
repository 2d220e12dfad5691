// C-ABI entry points of librib: host-side validation, error reporting and the
// launches of the kernels in the other translation units. No entry point
// allocates device memory or synchronises (except rib_device_error, whose job
// is to synchronise and read the device error word).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <initializer_list>
#include <mutex>
#include <string>

#include "rib_internal.h"

namespace rib {

namespace {
thread_local std::string g_msg;
__device__ int g_device_error;   // site code of the first bounded wait that ran out

constexpr int kMaxDevices = 64;
void* g_sym_addr[kSymSlots][kMaxDevices] = {{nullptr}};
int g_sms[kMaxDevices] = {0};
std::mutex g_mu;

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeFn g_encode = nullptr;

int current_device() {
  int d = 0;
  cudaGetDevice(&d);
  return d;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Every pointer in the list aligned to `a` bytes (null pointers pass; they
// are checked separately where they are not allowed).
bool all_aligned(std::initializer_list<const void*> ps, size_t a) {
  for (const void* p : ps)
    if (!aligned(p, a)) return false;
  return true;
}

const char* site_name(int s) {
  switch (s) {
    case 101: return "attention: Q tiles";
    case 102: return "attention: free K/V stage";
    case 103: return "attention: K/V stage loaded";
    case 104: return "attention: S read by softmax";
    case 105: return "attention: P written by softmax";
    case 106: return "attention: S ready";
    case 107: return "attention: P.V ready";
    case 108: return "attention: final MMA drain";
    case 109: return "attention: TMA drain";
    case 201: return "token GEMM: raw stage free";
    case 202: return "token GEMM: raw stage loaded";
    case 203: return "token GEMM: A operand free";
    case 204: return "token GEMM: A operand written";
    case 205: return "token GEMM: accumulator free";
    case 206: return "token GEMM: accumulator ready";
    case 207: return "token GEMM: drain";
    case 208: return "token GEMM: weights staged";
    case 301: return "attention backward: own tile";
    case 302: return "attention backward: stage loaded";
    case 303: return "attention backward: free stage";
    case 304: return "attention backward: S read";
    case 305: return "attention backward: dS written";
    case 306: return "attention backward: S ready";
    case 307: return "attention backward: accumulate MMAs";
    case 308: return "attention backward: final MMA drain";
    case 309: return "attention backward: TMA drain";
    case 901: return "self-test wait (nothing arrives)";
    default: return "unknown";
  }
}
}  // namespace

void set_error(const std::string& msg) { g_msg = msg; }

rib_status fail(rib_status s, const std::string& msg) {
  g_msg = msg;
  return s;
}

rib_status cuda_fail(cudaError_t e, const char* what) {
  char buf[256];
  std::snprintf(buf, sizeof(buf), "%s: %s (%d)", what, cudaGetErrorString(e), static_cast<int>(e));
  g_msg = buf;
  return RIB_ERR_CUDA;
}

int* device_error_word() {
  cudaError_t e;
  return static_cast<int*>(cached_symbol_address(kSymErrorWord, &g_device_error, &e));
}

void* cached_symbol_address(int slot, const void* symbol, cudaError_t* err) {
  *err = cudaSuccess;
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices || slot < 0 || slot >= kSymSlots) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sym_addr[slot][d]) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, symbol);
    if (*err != cudaSuccess) return nullptr;
    g_sym_addr[slot][d] = p;
  }
  return g_sym_addr[slot][d];
}

int sm_count() {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sms[d]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d);
    g_sms[d] = n > 0 ? n : 148;
  }
  return g_sms[d];
}

CUresult encode_tiled(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t rank, void* addr, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return CUDA_ERROR_NOT_FOUND;
      g_encode = reinterpret_cast<EncodeFn>(fn);
    }
  }
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return g_encode(map, dtype, rank, addr, reinterpret_cast<const cuuint64_t*>(dims),
                  reinterpret_cast<const cuuint64_t*>(strides_bytes), reinterpret_cast<const cuuint32_t*>(box), estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

bool window_tiling(int M, WindowTiling* t) {
  if (M < 16 || M > 256 || M % 16 != 0) return false;
  for (int tc = 128; tc >= 16; tc /= 2) {
    const int tr = 128 / tc;
    if (M % tc == 0 && M % tr == 0) {
      t->tc = tc;
      t->tr = tr;
      return true;
    }
  }
  return false;
}

rib_status check_gate_args(const char* who, const void* X, rib_dtype xdtype, int B, int H, int W, int C,
                           const float* Wdw, const float* bdw, const void* Wpw, const float* bpw, const void* sig_gate) {
  char buf[200];
  auto bad = [&](rib_status st, const char* what) {
    std::snprintf(buf, sizeof(buf), "%s: %s", who, what);
    return fail(st, buf);
  };
  if (!X || !Wdw || !bdw || !Wpw || !bpw || !sig_gate) return bad(RIB_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || H <= 0 || W <= 0 || C <= 0) return bad(RIB_ERR_INVALID_ARG, "sizes must be positive");
  if (C % 4 || C > 256) return bad(RIB_ERR_UNSUPPORTED, "needs C % 4 == 0 and C <= 256");
  if (xdtype != RIB_BF16 && xdtype != RIB_F16)
    return bad(RIB_ERR_UNSUPPORTED, "X must be bf16 or fp16 (convert f32 maps with rib_f32_to_bf16)");
  if (!aligned(sig_gate, 16)) return bad(RIB_ERR_ALIGNMENT, "sig_gate needs 16-byte alignment");
  if (!aligned(X, 8)) return bad(RIB_ERR_ALIGNMENT, "X needs 8-byte alignment");
  if (!all_aligned({Wdw, bdw, bpw}, 4) || !aligned(Wpw, 2))
    return bad(RIB_ERR_ALIGNMENT, "fp32 weights 4-byte, Wpw 2-byte aligned");
  return RIB_OK;
}

rib_status cla_gate_two_pass(const char* who, const void* X, int B, int H, int W, int C, const float* Wdw,
                             const float* bdw, const void* Wpw, const float* bpw, void* sig_gate, void* D,
                             cudaStream_t stream) {
  char buf[200];
  if (!aligned(X, 16) || !aligned(D, 16)) {
    std::snprintf(buf, sizeof(buf), "%s: the two-pass gate needs X and its depthwise buffer 16-byte aligned", who);
    return fail(RIB_ERR_ALIGNMENT, buf);
  }
  cudaError_t e = launch_dwconv3x3(X, Wdw, bdw, D, B, H, W, C, stream);
  if (e != cudaSuccess) {
    std::snprintf(buf, sizeof(buf), "%s: depthwise launch", who);
    return cuda_fail(e, buf);
  }
  GemmLaunch g{};
  g.A = D;
  g.B = B;
  g.H = H;
  g.W = W;
  g.Hp = H;
  g.Wp = W;
  g.K = C;
  g.mode = 1;
  g.n_real = C;
  g.w_cols = C;
  g.njobs = 1;
  g.jobs[0] = GemmJob{Wpw, sig_gate, (C + 15) / 16 * 16, 0, 0, -1, 1.0f, bpw};
  e = launch_token_gemm(g, stream);
  if (e != cudaSuccess) {
    std::snprintf(buf, sizeof(buf), "%s: pointwise launch", who);
    return cuda_fail(e, buf);
  }
  return RIB_OK;
}

}  // namespace rib

using namespace rib;

extern "C" {

const char* rib_last_error(void) { return g_msg.c_str(); }

int rib_version(void) { return 202; }

rib_status rib_device_error(cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "rib_device_error: stream synchronise");
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "rib_device_error: read error word");
  if (v != 0) {
    const int zero = 0;
    cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
    char buf[160];
    std::snprintf(buf, sizeof(buf), "device wait timed out at site %d (%s)", v, site_name(v));
    return fail(RIB_ERR_TIMEOUT, buf);
  }
  g_msg.clear();
  return RIB_OK;
}

int rib_head_pad(int C, int heads) {
  if (heads <= 0 || C <= 0 || C % heads) return -1;
  const int dh = C / heads;
  return (dh + 15) / 16 * 16;
}

size_t rib_pos_cache_bytes(const rib_mlp_desc* m, int window) {
  if (!m || window <= 0) return 0;
  return static_cast<size_t>(m->heads) * window * window * m->R * 2;
}

rib_status rib_pos_encode(const rib_mlp_desc* m, int window, void* qp, void* kp, size_t cache_bytes,
                          cudaStream_t stream) {
  if (!m || !qp || !kp || !m->Wh || !m->bh || !m->Wpq || !m->Wpk)
    return fail(RIB_ERR_INVALID_ARG, "rib_pos_encode: null pointer");
  if (m->L < 1 || m->L > 16 || m->hidden < 1 || m->hidden > 256 || m->heads < 1 || m->heads > 16 || window < 1 ||
      window > 256)
    return fail(RIB_ERR_INVALID_ARG, "rib_pos_encode: L in 1..16, hidden 1..256, heads 1..16, window 1..256");
  if (m->R != 16) return fail(RIB_ERR_UNSUPPORTED, "rib_pos_encode: R must be 16");
  if (cache_bytes < rib_pos_cache_bytes(m, window))
    return fail(RIB_ERR_INVALID_ARG, "rib_pos_encode: cache_bytes smaller than rib_pos_cache_bytes()");
  if (!aligned(qp, 16) || !aligned(kp, 16)) return fail(RIB_ERR_ALIGNMENT, "rib_pos_encode: caches need 16-byte alignment");
  if (!all_aligned({m->Wh, m->bh, m->Wpq, m->Wpk}, 4))
    return fail(RIB_ERR_ALIGNMENT, "rib_pos_encode: MLP weights need 4-byte alignment");
  cudaError_t e = launch_pos_encode(*m, window, qp, kp, stream);
  if (e != cudaSuccess) return cuda_fail(e, "rib_pos_encode launch");
  return RIB_OK;
}

rib_status rib_f32_to_bf16(const float* x, void* y, size_t n, cudaStream_t stream) {
  if ((!x || !y) && n) return fail(RIB_ERR_INVALID_ARG, "rib_f32_to_bf16: null pointer");
  if (!aligned(x, 16) || !aligned(y, 8)) return fail(RIB_ERR_ALIGNMENT, "rib_f32_to_bf16: x 16-byte, y 8-byte aligned");
  cudaError_t e = launch_f32_to_bf16(x, y, n, stream);
  if (e != cudaSuccess) return cuda_fail(e, "rib_f32_to_bf16 launch");
  return RIB_OK;
}

rib_status rib_bf16_to_f32(const void* x, float* y, size_t n, cudaStream_t stream) {
  if ((!x || !y) && n) return fail(RIB_ERR_INVALID_ARG, "rib_bf16_to_f32: null pointer");
  if (!aligned(x, 8) || !aligned(y, 16)) return fail(RIB_ERR_ALIGNMENT, "rib_bf16_to_f32: x 8-byte, y 16-byte aligned");
  cudaError_t e = launch_bf16_to_f32(x, y, n, stream);
  if (e != cudaSuccess) return cuda_fail(e, "rib_bf16_to_f32 launch");
  return RIB_OK;
}

rib_status rib_qkv_project(const void* X, rib_dtype xdtype, int B, int H, int W, int C, int heads, int window,
                           const void* Wq, const void* Wk, const void* Wv, float q_scale, void* Qc, void* Kc, void* V,
                           cudaStream_t stream) {
  if (!X || !Wq || !Wk || !Wv || !Qc || !Kc || !V) return fail(RIB_ERR_INVALID_ARG, "rib_qkv_project: null pointer");
  if (B <= 0 || H <= 0 || W <= 0 || C <= 0 || heads <= 0 || C % heads || window <= 0)
    return fail(RIB_ERR_INVALID_ARG, "rib_qkv_project: sizes must be positive and C % heads == 0");
  const int dh = C / heads, DP = rib_head_pad(C, heads);
  if (dh % 2 || dh > 30 || C > 256 || C % 4 || heads * DP > 256 || heads * 32 > 256)
    return fail(RIB_ERR_UNSUPPORTED, "rib_qkv_project: needs dh even and <= 30, C <= 256, C % 4 == 0, heads <= 8");
  if (xdtype != RIB_BF16 && xdtype != RIB_F16)
    return fail(RIB_ERR_UNSUPPORTED, "rib_qkv_project: X must be bf16 or fp16 (convert f32 maps with rib_f32_to_bf16)");
  if (!aligned(X, 8) || !aligned(Qc, 16) || !aligned(Kc, 16) || !aligned(V, 16))
    return fail(RIB_ERR_ALIGNMENT, "rib_qkv_project: X 8-byte, outputs 16-byte aligned");
  if (!all_aligned({Wq, Wk, Wv}, 2)) return fail(RIB_ERR_ALIGNMENT, "rib_qkv_project: weights need 2-byte alignment");
  GemmLaunch g{};
  g.A = X;
  g.B = B;
  g.H = H;
  g.W = W;
  g.Hp = (H + window - 1) / window * window;
  g.Wp = (W + window - 1) / window * window;
  g.K = C;
  g.a_f16 = xdtype == RIB_F16 ? 1 : 0;
  g.mode = 0;
  g.heads = heads;
  g.dh = dh;
  g.w_cols = C;
  g.njobs = 3;
  g.jobs[0] = GemmJob{Wq, Qc, heads * DP, DP, 0, -1, q_scale, nullptr};
  // Kc's columns d >= dh are 1 for every key when the head is padded (dh <
  // DP): the attention kernels carry each query row's softmax reference (the
  // forward) and log-sum-exp (the backward) through them; V's columns d >= dh
  // are 1 (the forward's softmax denominator, the backward's D)
  g.jobs[1] = GemmJob{Wk, Kc, heads * DP, DP, 0, dh < DP ? dh : -1, 1.0f, nullptr};
  g.jobs[2] = GemmJob{Wv, V, heads * 32, 32, 0, dh, 1.0f, nullptr};
  cudaError_t e = launch_token_gemm(g, stream);
  if (e != cudaSuccess) return cuda_fail(e, "rib_qkv_project launch");
  return RIB_OK;
}

size_t cla_gate_workspace_size(int B, int H, int W, int C) {
  if (B <= 0 || H <= 0 || W <= 0 || C <= 0) return 0;
  return static_cast<size_t>(B) * H * W * C * 2;
}

rib_status cla_gate(const void* X, rib_dtype xdtype, int B, int H, int W, int C, const float* Wdw, const float* bdw,
                    const void* Wpw, const float* bpw, void* sig_gate, void* ws, size_t ws_bytes,
                    cudaStream_t stream) {
  rib_status st = check_gate_args("cla_gate", X, xdtype, B, H, W, C, Wdw, bdw, Wpw, bpw, sig_gate);
  if (st != RIB_OK) return st;
  if (ws && ws_bytes < cla_gate_workspace_size(B, H, W, C))
    return fail(RIB_ERR_INVALID_ARG, "cla_gate: workspace too small");
  if (ws && !aligned(ws, 16)) return fail(RIB_ERR_ALIGNMENT, "cla_gate: the workspace needs 16-byte alignment");
  if (cla_gate_fused_supported(X, B, H, W, C)) {
    // one pass: depthwise into the pointwise GEMM's operand tile; the
    // depthwise output reaches the workspace only when one is given
    cudaError_t e = launch_cla_gate_fused(X, xdtype == RIB_F16 ? 1 : 0, Wdw, bdw, Wpw, bpw, sig_gate, ws, B, H, W, C,
                                          stream);
    if (e != cudaSuccess) return cuda_fail(e, "cla_gate: fused launch");
    return RIB_OK;
  }
  // two passes through the workspace: maps whose rows of lines the fused
  // kernel's tensor map cannot describe (W*C % 8 != 0) or an X that is not
  // 16-byte aligned
  if (xdtype == RIB_F16)
    return fail(RIB_ERR_UNSUPPORTED, "cla_gate: fp16 maps need W*C % 8 == 0 and a 16-byte aligned X");
  if (!ws)
    return fail(RIB_ERR_INVALID_ARG,
                "cla_gate: this map (W*C % 8 != 0 or X not 16-byte aligned) needs the workspace");
  return cla_gate_two_pass("cla_gate", X, B, H, W, C, Wdw, bdw, Wpw, bpw, sig_gate, ws, stream);
}

size_t rib_conv_ffn_workspace_size(int B, int H, int W, int hidden) {
  if (B <= 0 || H <= 0 || W <= 0 || hidden <= 0) return 0;
  return static_cast<size_t>(B) * H * W * ((hidden + 7) / 8 * 8) * 2;
}

rib_status rib_conv_ffn(const void* xn, rib_dtype xndtype, float* x, int B, int H, int W, int C, int hidden, const void* W1,
                        const float* b1, const float* Wf, const float* bf, const void* W2, const float* b2, void* ws,
                        size_t ws_bytes, cudaStream_t stream) {
  if (!xn || !x || !W1 || !b1 || !Wf || !bf || !W2 || !b2 || !ws)
    return fail(RIB_ERR_INVALID_ARG, "rib_conv_ffn: null pointer");
  if (B <= 0 || H <= 0 || W <= 0 || C <= 0 || hidden <= 0)
    return fail(RIB_ERR_INVALID_ARG, "rib_conv_ffn: sizes must be positive");
  if (C % 4 || C > 256 || hidden > 256)
    return fail(RIB_ERR_UNSUPPORTED, "rib_conv_ffn: needs C % 4 == 0, C <= 256 and hidden <= 256");
  if (xndtype != RIB_BF16 && xndtype != RIB_F16)
    return fail(RIB_ERR_UNSUPPORTED, "rib_conv_ffn: xn must be bf16 or fp16");
  if (ws_bytes < rib_conv_ffn_workspace_size(B, H, W, hidden))
    return fail(RIB_ERR_INVALID_ARG, "rib_conv_ffn: workspace too small");
  if (!aligned(xn, 8) || !aligned(x, 16) || !aligned(ws, 16))
    return fail(RIB_ERR_ALIGNMENT, "rib_conv_ffn: xn 8-byte, x and workspace 16-byte aligned");
  if (!all_aligned({b1, Wf, bf, b2}, 4) || !all_aligned({W1, W2}, 2))
    return fail(RIB_ERR_ALIGNMENT, "rib_conv_ffn: fp32 weights 4-byte, bf16 weights 2-byte aligned");
  const int HP = (hidden + 7) / 8 * 8;   // hidden channels as stored (the padding is zero)
  // h = GELU(xn W1 + b1): token GEMM with the GELU epilogue
  GemmLaunch g{};
  g.A = xn;
  g.B = B;
  g.H = H;
  g.W = W;
  g.Hp = H;
  g.Wp = W;
  g.K = C;
  g.mode = 1;
  g.gelu = 1;
  g.a_f16 = xndtype == RIB_F16 ? 1 : 0;
  g.n_real = HP;
  g.n_valid = hidden;
  g.w_cols = hidden;
  g.njobs = 1;
  // fp16 hidden features (saturating): see the second step
  g.jobs[0] = GemmJob{W1, ws, (hidden + 15) / 16 * 16, 0, 1, -1, 1.0f, b1};
  cudaError_t e = launch_token_gemm(g, stream);
  if (e == cudaErrorInvalidConfiguration)
    return fail(RIB_ERR_UNSUPPORTED, "rib_conv_ffn: C and hidden too wide for the first linear map's shared memory");
  if (e != cudaSuccess) return cuda_fail(e, "rib_conv_ffn: first linear map launch");
  // x += (h + DWConv3x3(h)) W2 + b2: depthwise into the pointwise operand tile
  if (!dw_pw_fused_supported(ws, W, HP, C))
    return fail(RIB_ERR_UNSUPPORTED, "rib_conv_ffn: map shape not supported by the depthwise-pointwise kernel");
  e = launch_dw_pw_fused(ws, B, H, W, HP, hidden, C, Wf, bf, W2, b2, nullptr, nullptr, x, 1, 1, stream);
  if (e != cudaSuccess) return cuda_fail(e, "rib_conv_ffn: depthwise and second linear map launch");
  return RIB_OK;
}

size_t rib_window_attention_workspace_size(const rib_attn_desc*) { return 0; }

rib_status rib_window_attention(const rib_attn_desc* d, const void* Qc, const void* Kc, const void* V,
                                const void* qp, const void* kp, const void* gate, const void* resid, void* Y,
                                float* lse, void* O_out, cudaStream_t stream) {
  if (!d || !Qc || !Kc || !V || !qp || !kp || !Y) return fail(RIB_ERR_INVALID_ARG, "rib_window_attention: null pointer");
  if (d->B <= 0 || d->H <= 0 || d->W <= 0 || d->C <= 0 || d->heads <= 0 || d->C % d->heads)
    return fail(RIB_ERR_INVALID_ARG, "rib_window_attention: sizes must be positive and C % heads == 0");
  const int dh = d->C / d->heads, DP = rib_head_pad(d->C, d->heads);
  if (d->R != 16) return fail(RIB_ERR_UNSUPPORTED, "rib_window_attention: R must be 16");
  if (dh % 2 || dh > 30) return fail(RIB_ERR_UNSUPPORTED, "rib_window_attention: needs dh even and <= 30");
  WindowTiling t;
  if (!window_tiling(d->window, &t))
    return fail(RIB_ERR_UNSUPPORTED, "rib_window_attention: window must be a multiple of 16 in 16..256");
  if (!(d->softmax_scale > 0.f) || !std::isfinite(d->softmax_scale))
    return fail(RIB_ERR_INVALID_ARG, "rib_window_attention: softmax_scale must be positive and finite");
  if (d->out_dtype != RIB_BF16 && d->out_dtype != RIB_F32 && d->out_dtype != RIB_F16)
    return fail(RIB_ERR_INVALID_ARG, "rib_window_attention: out_dtype must be RIB_BF16, RIB_F32 or RIB_F16");
  const void* ptrs[] = {Qc, Kc, V, qp, kp, gate, resid, Y, lse, O_out};
  for (const void* p : ptrs)
    if (p && !aligned(p, 16)) return fail(RIB_ERR_ALIGNMENT, "rib_window_attention: tensors need 16-byte alignment");
  AttnLaunch a{};
  a.B = d->B; a.H = d->H; a.W = d->W; a.C = d->C; a.heads = d->heads; a.dh = dh; a.DP = DP; a.M = d->window;
  a.tc = t.tc; a.tr = t.tr;
  a.scale_log2 = d->softmax_scale * 1.4426950408889634f;
  a.mask_padding = d->mask_padding ? 1 : 0;
  a.out_f32 = d->out_dtype == RIB_F32 ? 1 : 0;
  a.out_f16 = d->out_dtype == RIB_F16 ? 1 : 0;
  a.Qc = Qc; a.Kc = Kc; a.V = V; a.qp = qp; a.kp = kp; a.gate = gate; a.resid = resid; a.Y = Y; a.lse = lse;
  a.O_out = O_out;
  cudaError_t e = launch_window_attention(a, stream);
  if (e != cudaSuccess) return cuda_fail(e, "rib_window_attention launch");
  return RIB_OK;
}

static rib_status check_attn_desc(const rib_attn_desc* d, const char* who, int* dh, int* DP, WindowTiling* t) {
  char buf[160];
  if (!d) {
    std::snprintf(buf, sizeof(buf), "%s: null descriptor", who);
    return fail(RIB_ERR_INVALID_ARG, buf);
  }
  if (d->B <= 0 || d->H <= 0 || d->W <= 0 || d->C <= 0 || d->heads <= 0 || d->C % d->heads) {
    std::snprintf(buf, sizeof(buf), "%s: sizes must be positive and C %% heads == 0", who);
    return fail(RIB_ERR_INVALID_ARG, buf);
  }
  *dh = d->C / d->heads;
  *DP = rib_head_pad(d->C, d->heads);
  if (d->R != 16 || *dh % 2 || *dh > 30 || !window_tiling(d->window, t)) {
    std::snprintf(buf, sizeof(buf), "%s: needs R == 16, dh even and <= 30, window a multiple of 16 in 16..256", who);
    return fail(RIB_ERR_UNSUPPORTED, buf);
  }
  if (!(d->softmax_scale > 0.f) || !std::isfinite(d->softmax_scale)) {
    std::snprintf(buf, sizeof(buf), "%s: softmax_scale must be positive and finite", who);
    return fail(RIB_ERR_INVALID_ARG, buf);
  }
  if (d->mask_padding) {
    std::snprintf(buf, sizeof(buf), "%s: the key-padding mask is forward only", who);
    return fail(RIB_ERR_UNSUPPORTED, buf);
  }
  return RIB_OK;
}

rib_status rib_attention_bwd_prep(const rib_attn_desc* d, const void* dY, const void* sig_gate, const void* O,
                                  void* dO, float* Dsum, void* dG, cudaStream_t stream) {
  int dh, DP;
  WindowTiling t;
  rib_status st = check_attn_desc(d, "rib_attention_bwd_prep", &dh, &DP, &t);
  if (st != RIB_OK) return st;
  if (!dY || !sig_gate || !O || !dO || !Dsum) return fail(RIB_ERR_INVALID_ARG, "rib_attention_bwd_prep: null pointer");
  if (!all_aligned({dY, sig_gate, dG, Dsum}, 4) || !all_aligned({O, dO}, 16))
    return fail(RIB_ERR_ALIGNMENT, "rib_attention_bwd_prep: dY, sig_gate, dG, Dsum 4-byte, O and dO 16-byte aligned");
  cudaError_t e = launch_bwd_prep(dY, sig_gate, O, dO, Dsum, dG, d->B, d->H, d->W, d->C, d->heads, d->window,
                                  d->softmax_scale, stream);
  if (e != cudaSuccess) return cuda_fail(e, "rib_attention_bwd_prep launch");
  return RIB_OK;
}

// Workspace of the backward: the per-window partials of dQp and dKp (fp32),
// then, for padded heads with two spare columns (dh + 2 <= DP), the folded Q''
// content and rank tensors (bf16, per padded token and head).
static size_t bwd_partials_bytes(const rib_attn_desc* d) {
  const size_t nwin = static_cast<size_t>(d->B) * ((d->H + d->window - 1) / d->window) * ((d->W + d->window - 1) / d->window);
  return 2 * nwin * d->heads * d->window * d->window * 16 * sizeof(float);
}

static size_t bwd_fold_bytes(const rib_attn_desc* d, size_t* qf_bytes) {
  *qf_bytes = 0;
  if (d->heads <= 0 || d->C % d->heads) return 0;
  const int dh = d->C / d->heads, DP = rib_head_pad(d->C, d->heads);
  if (dh + 2 > DP) return 0;
  const size_t Tp = static_cast<size_t>(d->B) * ((d->H + d->window - 1) / d->window * d->window) *
                    ((d->W + d->window - 1) / d->window * d->window);
  *qf_bytes = Tp * d->heads * DP * 2;
  return *qf_bytes + Tp * d->heads * 16 * 2;
}

size_t rib_window_attention_bwd_workspace_size(const rib_attn_desc* d) {
  if (!d || d->window <= 0 || d->B <= 0 || d->H <= 0 || d->W <= 0) return 0;
  size_t qf;
  return bwd_partials_bytes(d) + bwd_fold_bytes(d, &qf);
}

rib_status rib_window_attention_bwd(const rib_attn_desc* d, const void* Qc, const void* Kc, const void* V,
                                    const void* qp, const void* kp, const float* lse, const void* dO,
                                    const float* Dsum, float* dQc, float* dKc, float* dV, float* dQp, float* dKp,
                                    void* ws, size_t ws_bytes, cudaStream_t stream) {
  int dh, DP;
  WindowTiling t;
  rib_status st = check_attn_desc(d, "rib_window_attention_bwd", &dh, &DP, &t);
  if (st != RIB_OK) return st;
  if (!Qc || !Kc || !V || !qp || !kp || !lse || !dO || !Dsum || !dQc || !dKc || !dV || !dQp || !dKp || !ws)
    return fail(RIB_ERR_INVALID_ARG, "rib_window_attention_bwd: null pointer");
  if (ws_bytes < rib_window_attention_bwd_workspace_size(d))
    return fail(RIB_ERR_INVALID_ARG, "rib_window_attention_bwd: workspace smaller than the workspace size query");
  const void* ptrs[] = {Qc, Kc, V, qp, kp, lse, dO, Dsum, dQc, dKc, dV, dQp, dKp, ws};
  for (const void* p : ptrs)
    if (!aligned(p, 16)) return fail(RIB_ERR_ALIGNMENT, "rib_window_attention_bwd: tensors need 16-byte alignment");
  AttnBwdLaunch a{};
  a.B = d->B; a.H = d->H; a.W = d->W; a.C = d->C; a.heads = d->heads; a.dh = dh; a.DP = DP; a.M = d->window;
  a.tc = t.tc; a.tr = t.tr;
  a.scale = d->softmax_scale;
  a.Qc = Qc; a.Kc = Kc; a.V = V; a.qp = qp; a.kp = kp; a.dO = dO; a.lse = lse;
  a.dQc = dQc; a.dKc = dKc; a.dV = dV; a.dQp = dQp; a.dKp = dKp;
  const size_t part = bwd_partials_bytes(d);
  a.ws_q = static_cast<float*>(ws);
  a.ws_k = a.ws_q + part / (2 * sizeof(float));
  size_t qf_bytes;
  if (bwd_fold_bytes(d, &qf_bytes) > 0) {
    a.qf = static_cast<uint8_t*>(ws) + part;
    a.qpf = static_cast<uint8_t*>(ws) + part + qf_bytes;
  }
  cudaError_t e = launch_window_attention_bwd(a, stream);
  if (e != cudaSuccess) return cuda_fail(e, "rib_window_attention_bwd launch");
  return RIB_OK;
}

size_t rib_qkv_project_bwd_workspace_size(int B, int H, int W, int C, int heads) {
  if (B <= 0 || H <= 0 || W <= 0 || C <= 0 || heads <= 0) return 0;
  return qkv_project_bwd_ws_bytes(B, H, W, C, heads);
}

rib_status rib_qkv_project_bwd(const void* X, rib_dtype xdtype, int B, int H, int W, int C, int heads, int window,
                               const void* Wq, const void* Wk, const void* Wv, float q_scale, const float* dQc,
                               const float* dKc, const float* dV, float* dX, float* dWq, float* dWk, float* dWv,
                               void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!X || !Wq || !Wk || !Wv || !dQc || !dKc || !dV || !dX || !dWq || !dWk || !dWv || !ws)
    return fail(RIB_ERR_INVALID_ARG, "rib_qkv_project_bwd: null pointer");
  if (B <= 0 || H <= 0 || W <= 0 || C <= 0 || heads <= 0 || C % heads || window <= 0)
    return fail(RIB_ERR_INVALID_ARG, "rib_qkv_project_bwd: sizes must be positive and C % heads == 0");
  const int dh = C / heads;
  if (dh % 2 || dh > 30 || C > 256 || C % 4 || heads * 32 > 256)
    return fail(RIB_ERR_UNSUPPORTED, "rib_qkv_project_bwd: needs dh even and <= 30, C <= 256, C % 4 == 0, heads <= 8");
  if (xdtype != RIB_BF16)
    return fail(RIB_ERR_UNSUPPORTED, "rib_qkv_project_bwd: the backward takes bf16 maps (convert with rib_f32_to_bf16)");
  if (!aligned(X, 8) || !aligned(dQc, 16) || !aligned(dKc, 16) || !aligned(dV, 16) || !aligned(dX, 16))
    return fail(RIB_ERR_ALIGNMENT, "rib_qkv_project_bwd: X 8-byte, gradients 16-byte aligned");
  if (!all_aligned({Wq, Wk, Wv}, 2) || !all_aligned({dWq, dWk, dWv}, 4))
    return fail(RIB_ERR_ALIGNMENT, "rib_qkv_project_bwd: weights 2-byte, weight gradients 4-byte aligned");
  if (ws_bytes < qkv_project_bwd_ws_bytes(B, H, W, C, heads))
    return fail(RIB_ERR_INVALID_ARG, "rib_qkv_project_bwd: workspace too small");
  if (!aligned(ws, 16)) return fail(RIB_ERR_ALIGNMENT, "rib_qkv_project_bwd: the workspace needs 16-byte alignment");
  QkvBwdLaunch a{};
  a.B = B;
  a.H = H;
  a.W = W;
  a.Hp = (H + window - 1) / window * window;
  a.Wp = (W + window - 1) / window * window;
  a.C = C;
  a.heads = heads;
  a.g[0] = dQc;
  a.g[1] = dKc;
  a.g[2] = dV;
  a.s[0] = q_scale;   // dQc is the gradient of the stored Qc = q_scale * X Wq
  a.s[1] = 1.f;
  a.s[2] = 1.f;
  a.Wt[0] = Wq;
  a.Wt[1] = Wk;
  a.Wt[2] = Wv;
  a.X = X;
  a.dX = dX;
  a.dW[0] = dWq;
  a.dW[1] = dWk;
  a.dW[2] = dWv;
  cudaError_t e = launch_qkv_project_bwd(a, ws, stream);
  if (e != cudaSuccess) return cuda_fail(e, "rib_qkv_project_bwd launch");
  return RIB_OK;
}

size_t cla_gate_bwd_workspace_size(int B, int H, int W, int C) {
  if (B <= 0 || H <= 0 || W <= 0 || C <= 0) return 0;
  return gate_bwd_ws_bytes(B, H, W, C);
}

rib_status cla_gate_bwd(const void* X, rib_dtype xdtype, int B, int H, int W, int C, const float* Wdw, const void* Wpw,
                        const void* D, const void* dG, float* dX, float* dWdw, float* dbdw, float* dWpw, float* dbpw,
                        void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!X || !Wdw || !Wpw || !D || !dG || !dX || !dWdw || !dbdw || !dWpw || !dbpw || !ws)
    return fail(RIB_ERR_INVALID_ARG, "cla_gate_bwd: null pointer");
  if (B <= 0 || H <= 0 || W <= 0 || C <= 0) return fail(RIB_ERR_INVALID_ARG, "cla_gate_bwd: sizes must be positive");
  if (C % 4 || C > 256) return fail(RIB_ERR_UNSUPPORTED, "cla_gate_bwd: needs C % 4 == 0 and C <= 256");
  if (xdtype != RIB_BF16)
    return fail(RIB_ERR_UNSUPPORTED, "cla_gate_bwd: the backward takes bf16 maps (convert with rib_f32_to_bf16)");
  if (ws_bytes < cla_gate_bwd_workspace_size(B, H, W, C))
    return fail(RIB_ERR_INVALID_ARG, "cla_gate_bwd: workspace too small");
  if (!aligned(X, 16) || !aligned(D, 16) || !aligned(dG, 16) || !aligned(dX, 16) || !aligned(ws, 16))
    return fail(RIB_ERR_ALIGNMENT, "cla_gate_bwd: X, D, dG, dX and workspace need 16-byte alignment");
  if (!all_aligned({Wdw, dWdw, dbdw, dWpw, dbpw}, 4) || !aligned(Wpw, 2))
    return fail(RIB_ERR_ALIGNMENT, "cla_gate_bwd: fp32 weights and gradients 4-byte, Wpw 2-byte aligned");
  GateBwdLaunch a{};
  a.B = B;
  a.H = H;
  a.W = W;
  a.C = C;
  a.X = X;
  a.Wdw = Wdw;
  a.Wpw = Wpw;
  a.D = D;
  a.dG = dG;
  a.dD = static_cast<float*>(ws);
  a.dX = dX;
  a.dWdw = dWdw;
  a.dbdw = dbdw;
  a.dWpw = dWpw;
  a.dbpw = dbpw;
  cudaError_t e = launch_cla_gate_bwd(a, ws, stream);
  if (e != cudaSuccess) return cuda_fail(e, "cla_gate_bwd launch");
  return RIB_OK;
}

size_t rib_pos_encode_bwd_workspace_size(const rib_mlp_desc* m, int window) {
  if (!m || window <= 0) return 0;
  // per token r, h, dpre; then the per-chunk partial sums of every weight
  const size_t per_token = static_cast<size_t>(window) * window * (2 + 4 * m->L + 2 * m->hidden);
  const size_t weights = 2 * static_cast<size_t>(m->hidden) * m->heads * m->R +
                         static_cast<size_t>(2 + 4 * m->L) * m->hidden + m->hidden;
  return (per_token + static_cast<size_t>(kPosBwdChunks) * weights) * sizeof(float);
}

rib_status rib_pos_encode_bwd(const rib_mlp_desc* m, int window, const float* dqp_cache, const float* dkp_cache,
                              float* dWh, float* dbh, float* dWpq, float* dWpk, void* ws, size_t ws_bytes,
                              cudaStream_t stream) {
  if (!m || !dqp_cache || !dkp_cache || !dWh || !dbh || !dWpq || !dWpk || !ws || !m->Wh || !m->bh || !m->Wpq || !m->Wpk)
    return fail(RIB_ERR_INVALID_ARG, "rib_pos_encode_bwd: null pointer");
  if (m->L < 1 || m->L > 16 || m->hidden < 1 || m->hidden > 256 || m->heads < 1 || m->heads > 16 || window < 1 ||
      window > 256)
    return fail(RIB_ERR_INVALID_ARG, "rib_pos_encode_bwd: L in 1..16, hidden 1..256, heads 1..16, window 1..256");
  if (m->R != 16) return fail(RIB_ERR_UNSUPPORTED, "rib_pos_encode_bwd: R must be 16");
  if (ws_bytes < rib_pos_encode_bwd_workspace_size(m, window))
    return fail(RIB_ERR_INVALID_ARG, "rib_pos_encode_bwd: workspace too small");
  if (!all_aligned({dqp_cache, dkp_cache, dWh, dbh, dWpq, dWpk, ws, m->Wh, m->bh, m->Wpq, m->Wpk}, 4))
    return fail(RIB_ERR_ALIGNMENT, "rib_pos_encode_bwd: fp32 tensors and workspace need 4-byte alignment");
  cudaError_t e = launch_pos_encode_bwd(*m, window, dqp_cache, dkp_cache, dWh, dbh, dWpq, dWpk, static_cast<float*>(ws),
                                        stream);
  if (e != cudaSuccess) return cuda_fail(e, "rib_pos_encode_bwd launch");
  return RIB_OK;
}

rib_status rib_layernorm(const void* x, rib_dtype xdtype, void* y, rib_dtype ydtype, int T, int C,
                         const float* gamma, const float* beta, float eps, cudaStream_t stream) {
  if (!x || !y) return fail(RIB_ERR_INVALID_ARG, "rib_layernorm: null pointer");
  if (T < 0 || C <= 0) return fail(RIB_ERR_INVALID_ARG, "rib_layernorm: sizes");
  if (C % 4 || C > 1024) return fail(RIB_ERR_UNSUPPORTED, "rib_layernorm: needs C % 4 == 0 and C <= 1024");
  if (!(eps > 0.f)) return fail(RIB_ERR_INVALID_ARG, "rib_layernorm: eps must be positive");
  if (xdtype != RIB_BF16 && xdtype != RIB_F32 && xdtype != RIB_F16)
    return fail(RIB_ERR_INVALID_ARG, "rib_layernorm: xdtype must be RIB_BF16, RIB_F32 or RIB_F16");
  if (ydtype != RIB_BF16 && ydtype != RIB_F16)
    return fail(RIB_ERR_INVALID_ARG, "rib_layernorm: ydtype must be RIB_BF16 or RIB_F16");
  if (!aligned(x, xdtype == RIB_F32 ? 16 : 8) || !aligned(y, 8))
    return fail(RIB_ERR_ALIGNMENT, "rib_layernorm: x 8-byte (16 for f32), y 8-byte aligned");
  if (!all_aligned({gamma, beta}, 4)) return fail(RIB_ERR_ALIGNMENT, "rib_layernorm: gamma and beta 4-byte aligned");
  cudaError_t e = launch_layernorm(x, xdtype == RIB_F32 ? 1 : (xdtype == RIB_F16 ? 2 : 0), y, ydtype == RIB_F16 ? 1 : 0,
                                   T, C, gamma, beta, eps, stream);
  if (e != cudaSuccess) return cuda_fail(e, "rib_layernorm launch");
  return RIB_OK;
}

}  // extern "C"
