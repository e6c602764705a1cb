// hy_kernels.h -- host-side launchers of the library's kernels (internal; the public
// C ABI is include/hymba.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

namespace hy {

// Raises `kernel`'s dynamic shared-memory limit to `bytes` once per device (devices 0..63);
// `done` is the kernel's own mask of devices already set.  Safe from several host threads
// (a repeated cudaFuncSetAttribute is harmless).
template <typename K>
cudaError_t smem_attr_once(K* kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const uint64_t bit = 1ull << dev;
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

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
  long long a_ld = 0;   // plain mode: row stride of A in elements (0: K)
  const void* x = nullptr;
  const void* meta = nullptr;
  int batch = 0, L = 0, n_meta = 0;
  int K = 0;
  // B operand W [N, K] row-major
  const void* w = nullptr;
  int N = 0;
  // Concatenated K (plain mode, bf16 only): C = [A | A2] [W | W2]^T, i.e. the product over
  // K columns of A and W followed by K2 columns of a2 [a_rows, K2] and w2 [N, K2] into the
  // same accumulator.  K2 = 0: off.
  const void* a2 = nullptr;
  const void* w2 = nullptr;
  int K2 = 0;
  // epilogue
  int epi = EPI_SEGMENTS;
  int nseg = 0;
  Seg seg[kMaxSegs];
  const void* resid = nullptr;
  long long resid_ld = 0;
  void* out = nullptr;
  long long out_ld = 0;
  // EPI_RESIDUAL and the fused branch-norm epilogue: resid and/or out in fp32 instead of
  // the GEMM's dtype (a residual stream carried in fp32)
  bool resid_f32 = false, out_f32 = false;
  // Output row remap (plain mode, segment epilogue): row r of A is written as row
  // (r / remap_L) * remap_T + remap_M + r % remap_L -- the user rows of [batch, L] landing
  // in a [batch, M + L] layout.  remap_L = 0: off.
  int remap_L = 0, remap_T = 0, remap_M = 0;
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
  // Final state: when set, h_out [batch, d_inner, d_state] fp32 receives each sequence's
  // state after its last row (what the next row of a generation step starts from).
  float* h_out = nullptr;
  // Start row: rows [t0, T) of each sequence are scanned (rows below t0 are neither read
  // nor written), from the state h0 [d_inner, d_state] fp32 of sequence b at
  // h0 + b * h0_bstride (h0_bstride 0: one state for every sequence); h0 NULL = zeros.
  int t0 = 0;
  const float* h0 = nullptr;
  long long h0_bstride = 0;
  // d_state 128 with the dt projection fused: scratch for the blocks' C B^T,
  // scan_mgram_bytes(s) bytes, 16-byte aligned (written and read within the call).
  void* mgram = nullptr;
};
cudaError_t launch_scan(const ScanDesc& s, cudaStream_t st);
// Bytes of ScanDesc::mgram the scan needs (0 when it needs none).
size_t scan_mgram_bytes(const ScanDesc& s);
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
  long long kv_rows = 0;  // rows per sequence in the K/V buffers (0: T; a cache may hold more)
  int q_row0 = 0;         // query rows below q_row0 need no output (their 128-row tiles are skipped)
};
cudaError_t launch_attention(const AttnDesc& a, cudaStream_t st);

// Generation step (decode.cu).  One query row per sequence at row `pos`; K/V cache
// rows of sequence b at (b * cap + row) * kv_ld; part: [batch, Hq, max_splits, dh + 2]
// fp32 partials; out at out + b * out_ld + h * dh.
struct DecodeAttnDesc {
  const void* q; const void* k; const void* v;
  long long cap, kv_ld;
  void* out; long long out_ld;
  float* part; int max_splits;
  int batch, n_q_heads, n_kv_heads, head_dim, pos, n_meta, window;
  bool bf16;
};
cudaError_t launch_attention_decode(const DecodeAttnDesc& a, cudaStream_t st);
// Number of key splits (and keys per split) the decode attention uses.
int decode_attn_splits(int batch, int n_kv_heads, int n_visible, int max_splits, int* keys_per_split);
// One scan step: h [batch, Di, N] fp32 updated in place; x, dt, gate [batch, Di];
// bc [batch, 2N] fp32; y at y + b * y_ld + c.
struct ScanStepDesc {
  const void* x; const void* dt; const float* bc; const void* gate; const float* a_log;
  bool a_per_state;
  float* h;
  void* y; long long y_ld;
  int batch, d_inner, d_state;
  bool bf16;
  const float* d_skip = nullptr;   // [Di]: y += D x before the gate, or nullptr
};
cudaError_t launch_scan_step(const ScanStepDesc& s, cudaStream_t st);

// z = [beta1 rms(z_a) || s2 beta2 rms(z_s)] in place (s2 = -1: difference fusion).
cudaError_t launch_branch_norm(void* z, const float* beta1, const float* beta2, long long rows, int w_attn,
                               int w_ssm, float eps, bool bf16, cudaStream_t st, float s2 = 1.f);
// The same per group of `group` (64, 128 or 256) features of each branch.
cudaError_t launch_group_norm(void* z, long long rows, int wa, int ws, int group, const float* beta1,
                              const float* beta2, float s2, float eps, bool bf16, cudaStream_t st);
// y = SiLU(bias + causal depthwise conv of width K of x) over [batch, Tseq, Di] rows.
cudaError_t launch_conv_silu(const void* x, const void* w, const float* bias, void* y, int batch, int Tseq, int Di,
                             int K, bool bf16, cudaStream_t st);
// z[r, c] += gate[r, c] * D[c] * x[r, c] for the SSM columns z (row stride z_ld).
cudaError_t launch_ssm_skip(void* z, long long z_ld, const void* gate, const void* x, const float* D, long long rows,
                            int Di, bool bf16, cudaStream_t st);
cudaError_t launch_rmsnorm(const void* x, void* y, long long rows, int d, float eps, bool bf16,
                           cudaStream_t st);
// Pre-norm of a residual stream kept in fp32: y = bf16(gain * x / sqrt(mean(x^2) + eps)) per
// row of x [rows, d] fp32 (gain [d] fp32, or NULL for unit gain); when y_lo is given it also
// receives the part of the fp32 result that the bf16 rounding dropped, bf16(v - float(y)).
cudaError_t launch_prenorm_f32(const float* x, const float* gain, void* y, void* y_lo, long long rows, int d,
                               float eps, cudaStream_t st, long long y_ld = 0);
// hi = bf16(src), lohi = [bf16(src - hi) | hi] per row: src [rows, cols] fp32, hi [rows, cols],
// lohi [rows, 2 cols] (bf16).
cudaError_t launch_split_hi_lo(const float* src, void* hi, void* lohi, int rows, int cols, cudaStream_t st);
cudaError_t launch_prenorm_f32_out_f32(const float* x, const float* gain, float* y, long long rows, int d, float eps,
                                       cudaStream_t st);
// h[b, t, :] = float([meta; x_b][t, :]) for a bf16 stack input (h fp32 [batch, L + M, d]).
cudaError_t launch_prepend_f32(const void* x, const void* meta, float* h, int batch, int L, int M, int d,
                               cudaStream_t st);
// dst + b * dst_stride = src for b in [0, batch): one block of `bytes` (a multiple of 16,
// 16-byte aligned addresses and stride) copied to every sequence.
cudaError_t launch_broadcast(const void* src, size_t bytes, void* dst, size_t dst_stride, int batch,
                             cudaStream_t st);
// dst[c, r] = src[r, c] for a bf16 matrix src [rows, cols] with row stride src_ld.
cudaError_t launch_transpose_bf16(const void* src, long long src_ld, void* dst, int rows, int cols,
                                  cudaStream_t st);
// Fused branch norm (bf16).  row_ssq: ssq[row] = (sum of z[row, :w_attn]^2, sum of
// z[row, w_attn:]^2).  scale_cols: w_out[n, k] = w[n, k] * (k < w_attn ? beta1[k] :
// beta2[k - w_attn]) for a [N, w_attn + w_ssm] weight.
cudaError_t launch_row_ssq(const void* z, long long rows, int w_attn, int w_ssm, float2* ssq, cudaStream_t st,
                           unsigned* status = nullptr);
cudaError_t launch_scale_cols(const void* w, void* w_out, int N, int w_attn, int w_ssm, const float* beta1,
                              const float* beta2, cudaStream_t st, float s2 = 1.f);

int num_sms();

}  // namespace hy
