// hy_kernels.h -- host-side launchers of the library's kernels (internal; the public
// C ABI is include/hymba.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace hy {

// Launch with programmatic stream serialization (see pdl_wait in hy_common.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// One column segment of a GEMM output: columns [col0, col1) of the product go to
// ptr + row * ld + (col - col0), optionally through an elementwise op.
enum SegOp : int { SEG_STORE = 0, SEG_SILU = 1, SEG_SOFTPLUS_BIAS = 2 };
struct Seg {
  int col0, col1;
  void* ptr;
  long long ld;
  int out_f32;         // 1: fp32 output, 0: the GEMM's dtype
  int op;              // SegOp
  const float* bias;   // SEG_SOFTPLUS_BIAS: bias[col - col0]
};
constexpr int kMaxSegs = 6;

enum EpiKind : int {
  EPI_SEGMENTS = 0,  // column segments (in_proj, x_proj, dt_proj, plain GEMMs)
  EPI_SWIGLU = 1,    // out[:, j] = SiLU(acc[:, j]) * acc[:, F + j]   (W rows: gate then up)
  EPI_RESIDUAL = 2   // out = resid + acc  (resid may alias out)
};

struct GemmDesc {
  // A operand: plain [a_rows, K] row-major, or "meta mode": the rows of
  // X~_b = [meta; x_b] for every sequence b, read straight from meta [M, K] and
  // x [batch, L, K] (the meta tokens are never copied).
  bool meta_mode = false;
  const void* a = nullptr;
  long long a_rows = 0;
  const void* x = nullptr;
  const void* meta = nullptr;
  int batch = 0, L = 0, n_meta = 0;
  int K = 0;
  // B operand W [N, K] row-major
  const void* w = nullptr;
  int N = 0;
  // epilogue
  int epi = EPI_SEGMENTS;
  int nseg = 0;
  Seg seg[kMaxSegs];
  const void* resid = nullptr;
  long long resid_ld = 0;
  void* out = nullptr;
  long long out_ld = 0;
  int swiglu_F = 0;
  // Fused branch norm (bf16 out_proj): the first dual_k_blocks 64-wide K blocks (the
  // attention columns of Z) accumulate apart from the rest (the SSM columns), and the
  // epilogue forms rsqrt(row_ssq.x * inv_wa + eps) acc_a + rsqrt(row_ssq.y * inv_ws + eps) acc_s.
  int dual_k_blocks = 0;
  const float2* row_ssq = nullptr;
  float inv_wa = 0.f, inv_ws = 0.f, eps = 0.f;
  unsigned* status = nullptr;
};

cudaError_t launch_gemm_bf16(const GemmDesc& g, cudaStream_t st);
cudaError_t launch_gemm_f32(const GemmDesc& g, cudaStream_t st);

struct ScanDesc {
  const void* x; const void* dt; const float* bc; const void* gate; const float* a_log;
  void* y; long long y_ld;
  int batch, T, d_inner, d_state;
  bool bf16;
  unsigned* status;
  bool a_per_state = false;  // a_log [d_inner, d_state] instead of [d_inner]
  // Fused dt projection (tensor-core scan only): when dt_low is set, dt is not read but
  // computed as softplus(dt_low w_dt^T + b_dt); dt_low [batch*T, dt_rank] bf16 (row
  // stride dt_rank), w_dt [d_inner, dt_rank] bf16, b_dt [d_inner] fp32.
  const void* dt_low = nullptr; const void* w_dt = nullptr; const float* b_dt = nullptr;
  int dt_rank = 0;
};
cudaError_t launch_scan(const ScanDesc& s, cudaStream_t st);
// The tensor-core form of the scan (bf16, d_state = 16, 16-byte aligned operands);
// cudaErrorNotSupported for any other configuration.
cudaError_t launch_scan_tc(const ScanDesc& s, cudaStream_t st);
// Whether launch_scan_tc takes this configuration with the dt projection fused
// (bf16, d_state 16, dt_rank 64, one decay per channel, 16-byte aligned operands).
bool scan_tc_fuses_dt(const ScanDesc& s);

struct AttnDesc {
  const void* q; long long q_ld;     // [batch*T, q_ld], head h at column h*dh
  const void* k; const void* v; long long kv_ld;  // [batch*T, kv_ld]
  void* out; long long out_ld;
  int batch, T, n_q_heads, n_kv_heads, head_dim, n_meta, window;
  bool bf16;
  unsigned* status;
};
cudaError_t launch_attention(const AttnDesc& a, cudaStream_t st);

cudaError_t launch_branch_norm(void* z, const float* beta1, const float* beta2, long long rows, int w_attn,
                               int w_ssm, float eps, bool bf16, cudaStream_t st);
cudaError_t launch_rmsnorm(const void* x, void* y, long long rows, int d, float eps, bool bf16,
                           cudaStream_t st);
// Fused branch norm (bf16).  row_ssq: ssq[row] = (sum of z[row, :w_attn]^2, sum of
// z[row, w_attn:]^2).  scale_cols: w_out[n, k] = w[n, k] * (k < w_attn ? beta1[k] :
// beta2[k - w_attn]) for a [N, w_attn + w_ssm] weight.
cudaError_t launch_row_ssq(const void* z, long long rows, int w_attn, int w_ssm, float2* ssq, cudaStream_t st);
cudaError_t launch_scale_cols(const void* w, void* w_out, int N, int w_attn, int w_ssm, const float* beta1,
                              const float* beta2, cudaStream_t st);

int num_sms();

}  // namespace hy
