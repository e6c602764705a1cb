// api.cu -- the C ABI (include/hymba.h): argument validation, workspace layout and
// the launch sequence of one hybrid-head layer and of a stack of blocks.
//
// Layer launch sequence (one stream; every step is a kernel of this library):
//   1 in_proj   X~ W_in^T -> Q | K | V | X_ssm | SiLU(G)   (meta rows read in place;
//               K/V go straight to kv_out for a producing layer)
//   2 x_proj    X_ssm W_x^T -> dt_low (dtype) | B, C (fp32)
//   3 dt_proj   softplus(dt_low W_dt^T + b_dt) -> dt
//   4 attention Q, K/V (own or kv_in) -> Z[:, :Hq*dh]
//   5 scan      x = X_ssm, dt, B, C, gate = SiLU(G) -> Z[:, Hq*dh:]
//   6 norm      Z <- [beta1 rms(Z_attn) || beta2 rms(Z_ssm)]   (in place; fp32 only)
//   7 out_proj  Z W_out^T -> out   (+ residual inside a stack)
// bf16 fuses the rewrite of step 6 away: each row's two sums of squares are read from
// Z, beta is folded into W_out's columns, and out_proj accumulates the attention and
// SSM columns apart and scales each by its row's 1 / rms.
#include <cstring>
#include <mutex>

#include "hy_common.cuh"
#include "hy_kernels.h"
#include "hymba.h"

namespace {

using hy::GemmDesc;
using hy::Seg;

inline size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
inline size_t esize(hymba_dtype_t t) { return t == HYMBA_BF16 ? 2 : 4; }

struct LayerWs {
  size_t q, kv, xs, g, dtlow, bc, dt, z, ssq, wsc, total;
};

// bf16 layers fuse the branch norm into out_proj (the row-sum kernel holds a row of up
// to 6144 bf16 in one warp's registers); fp32 layers run the separate norm kernel.
bool fused_branch_norm(const hymba_cfg_t& c) {
  return c.dtype == HYMBA_BF16 && c.n_q_heads * c.head_dim + c.d_inner <= 6144;
}

LayerWs layer_ws(const hymba_cfg_t& c, size_t base) {
  const size_t es = esize(c.dtype);
  const size_t rows = static_cast<size_t>(c.batch) * (c.seq_len + c.n_meta);
  const size_t wa = static_cast<size_t>(c.n_q_heads) * c.head_dim;
  const size_t wkv = static_cast<size_t>(c.n_kv_heads) * c.head_dim;
  LayerWs w;
  size_t o = base;
  w.q = o; o = al256(o + rows * wa * es);
  w.kv = o; o = al256(o + (c.kv_mode == HYMBA_KV_OWN ? 2 * rows * wkv * es : 0));
  w.xs = o; o = al256(o + rows * c.d_inner * es);
  w.g = o; o = al256(o + rows * c.d_inner * es);
  w.dtlow = o; o = al256(o + rows * c.dt_rank * es);
  w.bc = o; o = al256(o + rows * 2 * c.d_state * 4);
  w.dt = o; o = al256(o + rows * c.d_inner * es);
  w.z = o; o = al256(o + rows * (wa + c.d_inner) * es);
  // fused branch norm (bf16): per row, the sums of squares of Y_attn and Y_ssm; and
  // W_out with beta1 | beta2 folded into its columns
  const bool fused = fused_branch_norm(c);
  w.ssq = o; o = al256(o + (fused ? rows * 2 * sizeof(float) : 0));
  w.wsc = o; o = al256(o + (fused ? static_cast<size_t>(c.d_model) * (wa + c.d_inner) * es : 0));
  w.total = o;
  return w;
}

bool valid_state(int n) { return n == 16 || n == 32 || n == 64 || n == 128 || n == 256; }

hymba_status_t validate_cfg(const hymba_cfg_t* c) {
  if (!c) return HYMBA_ERR_INVALID_ARG;
  if (c->dtype != HYMBA_BF16 && c->dtype != HYMBA_F32) return HYMBA_ERR_INVALID_ARG;
  if (c->batch < 1 || c->seq_len < 1 || c->n_meta < 0 || c->d_model < 1 || c->n_q_heads < 1 ||
      c->n_kv_heads < 1 || c->head_dim < 1 || c->window < -1 || c->d_inner < 1 || c->d_state < 1 ||
      c->dt_rank < 1 || c->ffn_dim < 0 || c->kv_mode < 0 || c->kv_mode > 2 || !(c->rms_eps >= 0.f))
    return HYMBA_ERR_INVALID_ARG;
  if (c->n_q_heads % c->n_kv_heads != 0) return HYMBA_ERR_INVALID_ARG;
  if (c->a_per_state != 0 && c->a_per_state != 1) return HYMBA_ERR_INVALID_ARG;
  if (!valid_state(c->d_state)) return HYMBA_ERR_UNSUPPORTED;
  const long long rows = static_cast<long long>(c->batch) * (c->seq_len + c->n_meta);
  if (rows > (1ll << 31) - 1) return HYMBA_ERR_UNSUPPORTED;
  if (c->d_model % 8 || c->d_inner % 16 || (c->n_q_heads * c->head_dim) % 8) return HYMBA_ERR_UNSUPPORTED;
  if (c->dtype == HYMBA_BF16) {
    if (c->head_dim != 128) return HYMBA_ERR_UNSUPPORTED;
    if (c->n_meta % 8) return HYMBA_ERR_UNSUPPORTED;
    if (c->dt_rank % 16) return HYMBA_ERR_UNSUPPORTED;
    if (c->ffn_dim % 128) return HYMBA_ERR_UNSUPPORTED;
  } else {
    if (c->head_dim > 128) return HYMBA_ERR_UNSUPPORTED;
  }
  return HYMBA_OK;
}

hymba_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? HYMBA_OK : HYMBA_ERR_CUDA; }

cudaError_t gemm(const GemmDesc& g, hymba_dtype_t t, cudaStream_t st) {
  return t == HYMBA_BF16 ? hy::launch_gemm_bf16(g, st) : hy::launch_gemm_f32(g, st);
}

Seg seg(int c0, int c1, void* ptr, long long ld, int out_f32, int op, const float* bias = nullptr) {
  Seg s;
  s.col0 = c0;
  s.col1 = c1;
  s.ptr = ptr;
  s.ld = ld;
  s.out_f32 = out_f32;
  s.op = op;
  s.bias = bias;
  return s;
}

bool weights_ok(const hymba_weights_t* w, const hymba_cfg_t& c, bool need_ffn) {
  if (!w || !w->w_in || !w->w_x || !w->w_dt || !w->w_out || !w->a_log || !w->b_dt || !w->beta1 || !w->beta2)
    return false;
  if (need_ffn && c.ffn_dim > 0 && (!w->w_gate_up || !w->w_down)) return false;
  return true;
}

// The attention heads and the SSM heads of a layer are independent until the branch
// norm: the attention runs on a second stream of the library's (one per device, made on
// first use), forked from the caller's stream after in_proj and joined back before the
// norm, so that its CTAs and the scan's fill the SMs together.
cudaStream_t side_stream() {
  static std::mutex mu;
  static cudaStream_t streams[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!streams[dev] && cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking) != cudaSuccess)
    streams[dev] = nullptr;
  return streams[dev];
}

// Joins the side stream back into the caller's stream once (at join() or on any return).
struct SideJoin {
  cudaStream_t st = nullptr;
  cudaEvent_t done = nullptr;
  cudaError_t join() {
    if (!done) return cudaSuccess;
    const cudaError_t e = cudaStreamWaitEvent(st, done, 0);
    cudaEventDestroy(done);
    done = nullptr;
    return e;
  }
  ~SideJoin() { join(); }
};

// One layer.  x: meta mode when meta != nullptr, else [rows, d] holding X~.
// resid_out: when true the out_proj adds into `out` (out = out + Z W_out^T).
hymba_status_t run_layer(const void* x, const void* meta, const hymba_weights_t& w, const hymba_cfg_t& c,
                         const void* kv_in, void* kv_out, void* out, bool resid_out, uint8_t* ws, unsigned* status,
                         cudaStream_t st, void* const* events = nullptr) {
  bool marks_ok = true;
  auto mark = [&](int i) {
    if (events && cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st) != cudaSuccess) marks_ok = false;
  };
  const LayerWs L = layer_ws(c, 0);
  const int T = c.seq_len + c.n_meta;
  const long long rows = static_cast<long long>(c.batch) * T;
  const int wa = c.n_q_heads * c.head_dim, wkv = c.n_kv_heads * c.head_dim, di = c.d_inner;
  const size_t es = esize(c.dtype);
  const int f32out = 0;
  void* q = ws + L.q;
  void* xs = ws + L.xs;
  void* g = ws + L.g;
  void* dtlow = ws + L.dtlow;
  float* bc = reinterpret_cast<float*>(ws + L.bc);
  void* dt = ws + L.dt;
  void* z = ws + L.z;

  hy::ScanDesc sd;
  sd.x = xs;
  sd.dt = dt;
  sd.bc = bc;
  sd.gate = g;
  sd.a_log = w.a_log;
  sd.y = static_cast<uint8_t*>(z) + wa * es;
  sd.y_ld = wa + di;
  sd.batch = c.batch;
  sd.T = T;
  sd.d_inner = di;
  sd.d_state = c.d_state;
  sd.bf16 = c.dtype == HYMBA_BF16;
  sd.status = status;
  sd.a_per_state = c.a_per_state != 0;
  // bf16 with d_state 16 and dt_rank 64: dt_proj runs inside the tensor-core scan
  // (dt = softplus(dt_low W_dt^T + b_dt) per block, never stored)
  {
    hy::ScanDesc f = sd;
    f.dt_low = dtlow;
    f.w_dt = w.w_dt;
    f.b_dt = w.b_dt;
    f.dt_rank = c.dt_rank;
    if (hy::scan_tc_fuses_dt(f)) sd = f;
  }
  const bool fused_dt = sd.dt_low != nullptr;
  // bf16: the branch norm is fused into out_proj -- the rows of Z are not rewritten;
  // their two sums of squares are read once, beta is folded into W_out's columns, and
  // out_proj applies the two 1 / rms row scales to its two accumulators
  const bool fused_norm = fused_branch_norm(c);
  float2* ssq = reinterpret_cast<float2*>(ws + L.ssq);
  void* w_out_scaled = ws + L.wsc;
  void* kvbuf = c.kv_mode == HYMBA_KV_PRODUCE ? kv_out : (c.kv_mode == HYMBA_KV_OWN ? ws + L.kv : nullptr);
  const void* kv_k = c.kv_mode == HYMBA_KV_CONSUME ? kv_in : kvbuf;
  const void* kv_v = static_cast<const uint8_t*>(kv_k) + static_cast<size_t>(rows) * wkv * es;

  // 1 in_proj
  mark(0);
  GemmDesc gi;
  if (meta) {
    gi.meta_mode = true;
    gi.x = x;
    gi.meta = meta;
    gi.batch = c.batch;
    gi.L = c.seq_len;
    gi.n_meta = c.n_meta;
  } else {
    gi.a = x;
    gi.a_rows = rows;
  }
  gi.K = c.d_model;
  gi.w = w.w_in;
  int col = 0;
  gi.seg[gi.nseg++] = seg(col, col + wa, q, wa, f32out, hy::SEG_STORE);
  col += wa;
  if (c.kv_mode != HYMBA_KV_CONSUME) {
    gi.seg[gi.nseg++] = seg(col, col + wkv, kvbuf, wkv, f32out, hy::SEG_STORE);
    col += wkv;
    gi.seg[gi.nseg++] = seg(col, col + wkv, static_cast<uint8_t*>(kvbuf) + static_cast<size_t>(rows) * wkv * es, wkv,
                            f32out, hy::SEG_STORE);
    col += wkv;
  }
  gi.seg[gi.nseg++] = seg(col, col + di, xs, di, f32out, hy::SEG_STORE);
  col += di;
  gi.seg[gi.nseg++] = seg(col, col + di, g, di, f32out, hy::SEG_SILU);
  col += di;
  gi.N = col;
  gi.status = status;
  cudaError_t e = gemm(gi, c.dtype, st);
  if (e != cudaSuccess) return HYMBA_ERR_CUDA;

  // 4 attention heads -> Z[:, :wa], on the side stream unless stage events are recorded
  // (then every stage runs in order on st)
  hy::AttnDesc ad;
  ad.q = q;
  ad.q_ld = wa;
  ad.k = kv_k;
  ad.v = kv_v;
  ad.kv_ld = wkv;
  ad.out = z;
  ad.out_ld = wa + di;
  ad.batch = c.batch;
  ad.T = T;
  ad.n_q_heads = c.n_q_heads;
  ad.n_kv_heads = c.n_kv_heads;
  ad.head_dim = c.head_dim;
  ad.n_meta = c.n_meta;
  ad.window = c.window;
  ad.bf16 = c.dtype == HYMBA_BF16;
  ad.status = status;
  cudaStream_t side = events ? nullptr : side_stream();
  SideJoin joiner;
  joiner.st = st;
  if (side) {
    cudaEvent_t forked = nullptr, done = nullptr;
    if (cudaEventCreateWithFlags(&forked, cudaEventDisableTiming) != cudaSuccess) return HYMBA_ERR_CUDA;
    const bool ok = cudaEventRecord(forked, st) == cudaSuccess && cudaStreamWaitEvent(side, forked, 0) == cudaSuccess;
    cudaEventDestroy(forked);
    if (!ok || cudaEventCreateWithFlags(&done, cudaEventDisableTiming) != cudaSuccess) return HYMBA_ERR_CUDA;
    const cudaError_t ea = hy::launch_attention(ad, side);
    if (cudaEventRecord(done, side) != cudaSuccess) {
      cudaEventDestroy(done);
      return HYMBA_ERR_CUDA;
    }
    joiner.done = done;
    if (ea != cudaSuccess) return HYMBA_ERR_CUDA;
  }

  // 2 x_proj
  mark(1);
  GemmDesc gx;
  gx.a = xs;
  gx.a_rows = rows;
  gx.K = di;
  gx.w = w.w_x;
  gx.N = c.dt_rank + 2 * c.d_state;
  gx.seg[gx.nseg++] = seg(0, c.dt_rank, dtlow, c.dt_rank, f32out, hy::SEG_STORE);
  gx.seg[gx.nseg++] = seg(c.dt_rank, gx.N, bc, 2 * c.d_state, 1, hy::SEG_STORE);
  gx.status = status;
  if ((e = gemm(gx, c.dtype, st)) != cudaSuccess) return HYMBA_ERR_CUDA;

  // 3 dt_proj with softplus(. + b_dt) (in the scan when fused_dt)
  mark(2);
  if (!fused_dt) {
    GemmDesc gd;
    gd.a = dtlow;
    gd.a_rows = rows;
    gd.K = c.dt_rank;
    gd.w = w.w_dt;
    gd.N = di;
    gd.seg[gd.nseg++] = seg(0, di, dt, di, f32out, hy::SEG_SOFTPLUS_BIAS, w.b_dt);
    gd.status = status;
    if ((e = gemm(gd, c.dtype, st)) != cudaSuccess) return HYMBA_ERR_CUDA;
  }

  mark(3);
  if (!side && (e = hy::launch_attention(ad, st)) != cudaSuccess) return HYMBA_ERR_CUDA;

  // 5 selective scan + gate -> Z[:, wa:]
  mark(4);
  e = hy::launch_scan(sd, st);
  if (joiner.join() != cudaSuccess || e != cudaSuccess) return HYMBA_ERR_CUDA;  // the norm reads all of Z

  // 6 per-branch RMSNorm and beta
  mark(5);
  if (fused_norm) {
    if ((e = hy::launch_scale_cols(w.w_out, w_out_scaled, c.d_model, wa, di, w.beta1, w.beta2, st)) != cudaSuccess ||
        (e = hy::launch_row_ssq(z, rows, wa, di, ssq, st)) != cudaSuccess)
      return HYMBA_ERR_CUDA;
  } else if ((e = hy::launch_branch_norm(z, w.beta1, w.beta2, rows, wa, di, c.rms_eps, c.dtype == HYMBA_BF16,
                                         st)) != cudaSuccess) {
    return HYMBA_ERR_CUDA;
  }

  // 7 out_proj
  mark(6);
  GemmDesc go;
  go.a = z;
  go.a_rows = rows;
  go.K = wa + di;
  go.w = fused_norm ? w_out_scaled : w.w_out;
  go.N = c.d_model;
  if (fused_norm) {
    go.dual_k_blocks = wa / 64;
    go.row_ssq = ssq;
    go.inv_wa = 1.f / static_cast<float>(wa);
    go.inv_ws = 1.f / static_cast<float>(di);
    go.eps = c.rms_eps;
    go.out = out;
    go.out_ld = c.d_model;
  }
  if (resid_out) {
    go.epi = hy::EPI_RESIDUAL;
    go.resid = out;
    go.resid_ld = c.d_model;
    go.out = out;
    go.out_ld = c.d_model;
  } else {
    go.seg[go.nseg++] = seg(0, c.d_model, out, c.d_model, f32out, hy::SEG_STORE);
  }
  go.status = status;
  if ((e = gemm(go, c.dtype, st)) != cudaSuccess) return HYMBA_ERR_CUDA;
  mark(7);
  return marks_ok ? HYMBA_OK : HYMBA_ERR_CUDA;
}

// h[b] = [meta; x[b]] (stack input), vectorised 16-byte copy.
__global__ void prepend_kernel(const uint4* __restrict__ x, const uint4* __restrict__ meta, uint4* __restrict__ h,
                               long long row_vecs, int L, int M, long long total) {
  hy::pdl_trigger();
  hy::pdl_wait();
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = i / row_vecs, e = i - row * row_vecs;
    const long long T = L + M;
    const long long b = row / T;
    const long long t = row - b * T;
    h[i] = t < M ? meta[t * row_vecs + e] : x[(b * L + (t - M)) * row_vecs + e];
  }
}

// ---- library-owned scratch for hymba_layer_fwd_noalloc
//
// One fixed block of device memory per GPU, reserved when the module loads on that
// device and held until the process exits.  Host code must not use the symbol's name
// as a pointer (on the host it names a stand-in object, not device memory): the device
// address comes from cudaGetSymbolAddress, looked up once per device with that device
// current and cached.
static __device__ __align__(256) uint8_t g_noalloc_scratch[HYMBA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxNoallocDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxNoallocDevices] = {};

// Device address of the scratch block on the current device (set up on first use).
cudaError_t noalloc_scratch(uint8_t** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxNoallocDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    if (!ptr) return cudaErrorInvalidSymbol;
    g_noalloc_addr[dev] = ptr;
  }
  *out = static_cast<uint8_t*>(g_noalloc_addr[dev]);
  return cudaSuccess;
}

}  // namespace

extern "C" {

const char* hymba_status_string(hymba_status_t s) {
  switch (s) {
    case HYMBA_OK: return "ok";
    case HYMBA_ERR_INVALID_ARG: return "invalid argument";
    case HYMBA_ERR_UNSUPPORTED: return "unsupported configuration";
    case HYMBA_ERR_WORKSPACE: return "workspace missing or too small";
    case HYMBA_ERR_CUDA: return "CUDA launch or runtime error";
    case HYMBA_ERR_TIMEOUT: return "a kernel's bounded wait timed out";
  }
  return "unknown status";
}

int hymba_layer_fuses_dt_proj(const hymba_cfg_t* cfg) {
  if (validate_cfg(cfg) != HYMBA_OK) return 0;
  // the same test run_layer makes, on 256-byte aligned workspace buffers and weights
  hy::ScanDesc f;
  f.x = f.gate = f.dt_low = f.w_dt = reinterpret_cast<const void*>(256);
  f.y = reinterpret_cast<void*>(256);
  f.bc = reinterpret_cast<const float*>(256);
  f.b_dt = reinterpret_cast<const float*>(256);
  f.y_ld = static_cast<long long>(cfg->n_q_heads) * cfg->head_dim + cfg->d_inner;
  f.d_inner = cfg->d_inner;
  f.d_state = cfg->d_state;
  f.dt_rank = cfg->dt_rank;
  f.bf16 = cfg->dtype == HYMBA_BF16;
  f.a_per_state = cfg->a_per_state != 0;
  return hy::scan_tc_fuses_dt(f) ? 1 : 0;
}

size_t hymba_workspace_size(const hymba_cfg_t* cfg) {
  if (validate_cfg(cfg) != HYMBA_OK) return 0;
  return 256 + layer_ws(*cfg, 0).total;
}

size_t hymba_stack_workspace_size(const hymba_cfg_t* cfgs, int n_layers) {
  if (!cfgs || n_layers < 1) return 0;
  size_t layer_max = 0;
  for (int i = 0; i < n_layers; ++i) {
    if (validate_cfg(&cfgs[i]) != HYMBA_OK) return 0;
    const size_t t = layer_ws(cfgs[i], 0).total;
    layer_max = t > layer_max ? t : layer_max;
  }
  const hymba_cfg_t& c = cfgs[0];
  const size_t es = esize(c.dtype);
  const size_t rows = static_cast<size_t>(c.batch) * (c.seq_len + c.n_meta);
  size_t kvw = 0, ffn = 0;
  for (int i = 0; i < n_layers; ++i) {
    const size_t w = static_cast<size_t>(cfgs[i].n_kv_heads) * cfgs[i].head_dim;
    kvw = w > kvw ? w : kvw;
    ffn = static_cast<size_t>(cfgs[i].ffn_dim) > ffn ? cfgs[i].ffn_dim : ffn;
  }
  return 256 + al256(layer_max) + al256(rows * c.d_model * es) + al256(2 * rows * kvw * es) + al256(rows * ffn * es);
}

hymba_status_t hymba_layer_fwd(const void* x, const void* meta, const hymba_weights_t* w, const hymba_cfg_t* cfg,
                               const void* kv_in, void* kv_out, void* out, void* workspace, size_t ws_bytes,
                               void* stream) {
  return hymba_layer_fwd_events(x, meta, w, cfg, kv_in, kv_out, out, workspace, ws_bytes, stream, nullptr);
}

hymba_status_t hymba_layer_fwd_events(const void* x, const void* meta, const hymba_weights_t* w,
                                      const hymba_cfg_t* cfg, const void* kv_in, void* kv_out, void* out,
                                      void* workspace, size_t ws_bytes, void* stream, void* const* events) {
  hymba_status_t s = validate_cfg(cfg);
  if (s != HYMBA_OK) return s;
  if (!x || !out || !weights_ok(w, *cfg, false)) return HYMBA_ERR_INVALID_ARG;
  if (cfg->kv_mode == HYMBA_KV_CONSUME && !kv_in) return HYMBA_ERR_INVALID_ARG;
  if (cfg->kv_mode == HYMBA_KV_PRODUCE && !kv_out) return HYMBA_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < hymba_workspace_size(cfg)) return HYMBA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255) return HYMBA_ERR_INVALID_ARG;
  if (events)
    for (int i = 0; i < 8; ++i)
      if (!events[i]) return HYMBA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned* status = static_cast<unsigned*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(unsigned), st) != cudaSuccess) return HYMBA_ERR_CUDA;
  return run_layer(x, cfg->n_meta > 0 ? meta : nullptr, *w, *cfg, kv_in, kv_out, out, false,
                   static_cast<uint8_t*>(workspace) + 256, status, st, events);
}

hymba_status_t hymba_layer_fwd_noalloc(const void* x, const void* meta, const hymba_weights_t* w,
                                       const hymba_cfg_t* cfg, const void* kv_in, void* kv_out, void* out,
                                       void* stream) {
  hymba_status_t s = validate_cfg(cfg);
  if (s != HYMBA_OK) return s;
  if (!x || !out || !weights_ok(w, *cfg, false)) return HYMBA_ERR_INVALID_ARG;
  if (cfg->kv_mode == HYMBA_KV_CONSUME && !kv_in) return HYMBA_ERR_INVALID_ARG;
  if (cfg->kv_mode == HYMBA_KV_PRODUCE && !kv_out) return HYMBA_ERR_INVALID_ARG;
  // the same layout hymba_layer_fwd uses: status word, then the layer's intermediates
  if (hymba_workspace_size(cfg) > HYMBA_NOALLOC_SCRATCH_BYTES) return HYMBA_ERR_WORKSPACE;
  uint8_t* scratch = nullptr;
  if (noalloc_scratch(&scratch) != cudaSuccess) return HYMBA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned* status = reinterpret_cast<unsigned*>(scratch);
  // the block keeps the previous call's contents: the status word must start at zero
  // (every intermediate is written before it is read)
  if (cudaMemsetAsync(status, 0, sizeof(unsigned), st) != cudaSuccess) return HYMBA_ERR_CUDA;
  return run_layer(x, cfg->n_meta > 0 ? meta : nullptr, *w, *cfg, kv_in, kv_out, out, false, scratch + 256, status,
                   st);
}

hymba_status_t hymba_stack_fwd(const void* x, const void* meta, const hymba_weights_t* w, const hymba_cfg_t* cfgs,
                               int n_layers, void* out, void* workspace, size_t ws_bytes, void* stream) {
  if (!cfgs || n_layers < 1 || !w || !x || !out) return HYMBA_ERR_INVALID_ARG;
  const hymba_cfg_t& c0 = cfgs[0];
  for (int i = 0; i < n_layers; ++i) {
    hymba_status_t s = validate_cfg(&cfgs[i]);
    if (s != HYMBA_OK) return s;
    const hymba_cfg_t& c = cfgs[i];
    if (c.batch != c0.batch || c.seq_len != c0.seq_len || c.n_meta != c0.n_meta || c.d_model != c0.d_model ||
        c.dtype != c0.dtype)
      return HYMBA_ERR_INVALID_ARG;
    if (!weights_ok(&w[i], c, true)) return HYMBA_ERR_INVALID_ARG;
    if (c.kv_mode == HYMBA_KV_CONSUME &&
        (i == 0 || cfgs[i - 1].kv_mode != HYMBA_KV_PRODUCE || cfgs[i - 1].n_kv_heads != c.n_kv_heads ||
         cfgs[i - 1].head_dim != c.head_dim))
      return HYMBA_ERR_INVALID_ARG;
  }
  if (c0.n_meta > 0 && !meta) return HYMBA_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < hymba_stack_workspace_size(cfgs, n_layers)) return HYMBA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255) return HYMBA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned* status = static_cast<unsigned*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(unsigned), st) != cudaSuccess) return HYMBA_ERR_CUDA;

  size_t layer_max = 0, kvw = 0;
  for (int i = 0; i < n_layers; ++i) {
    const size_t t = layer_ws(cfgs[i], 0).total;
    layer_max = t > layer_max ? t : layer_max;
    const size_t k = static_cast<size_t>(cfgs[i].n_kv_heads) * cfgs[i].head_dim;
    kvw = k > kvw ? k : kvw;
  }
  const size_t es = esize(c0.dtype);
  const int T = c0.seq_len + c0.n_meta;
  const long long rows = static_cast<long long>(c0.batch) * T;
  uint8_t* base = static_cast<uint8_t*>(workspace) + 256;
  uint8_t* lws = base;
  uint8_t* xn = lws + al256(layer_max);
  uint8_t* kv = xn + al256(rows * c0.d_model * es);
  uint8_t* act = kv + al256(2 * rows * kvw * es);
  const bool bf16 = c0.dtype == HYMBA_BF16;

  // h = [meta; x] lives in `out` and is updated in place
  {
    const long long row_vecs = static_cast<long long>(c0.d_model) * es / 16;
    const long long total = rows * row_vecs;
    if (c0.d_model * es % 16) return HYMBA_ERR_UNSUPPORTED;
    const int blocks = static_cast<int>(total / 256 + 1 < 4096 ? total / 256 + 1 : 4096);
    if (hy::launch(prepend_kernel, dim3(blocks), dim3(256), 0, st, static_cast<const uint4*>(x),
                   static_cast<const uint4*>(meta), static_cast<uint4*>(out), row_vecs, c0.seq_len, c0.n_meta,
                   total) != cudaSuccess)
      return HYMBA_ERR_CUDA;
  }
  for (int i = 0; i < n_layers; ++i) {
    const hymba_cfg_t& c = cfgs[i];
    cudaError_t e = hy::launch_rmsnorm(out, xn, rows, c.d_model, c.rms_eps, bf16, st);
    if (e != cudaSuccess) return HYMBA_ERR_CUDA;
    hymba_status_t s = run_layer(xn, nullptr, w[i], c, kv, kv, out, true, lws, status, st);
    if (s != HYMBA_OK) return s;
    if (c.ffn_dim > 0) {
      if ((e = hy::launch_rmsnorm(out, xn, rows, c.d_model, c.rms_eps, bf16, st)) != cudaSuccess)
        return HYMBA_ERR_CUDA;
      GemmDesc gu;
      gu.a = xn;
      gu.a_rows = rows;
      gu.K = c.d_model;
      gu.w = w[i].w_gate_up;
      gu.N = 2 * c.ffn_dim;
      gu.epi = hy::EPI_SWIGLU;
      gu.swiglu_F = c.ffn_dim;
      gu.out = act;
      gu.out_ld = c.ffn_dim;
      gu.status = status;
      if (gemm(gu, c.dtype, st) != cudaSuccess) return HYMBA_ERR_CUDA;
      GemmDesc gdn;
      gdn.a = act;
      gdn.a_rows = rows;
      gdn.K = c.ffn_dim;
      gdn.w = w[i].w_down;
      gdn.N = c.d_model;
      gdn.epi = hy::EPI_RESIDUAL;
      gdn.resid = out;
      gdn.resid_ld = c.d_model;
      gdn.out = out;
      gdn.out_ld = c.d_model;
      gdn.status = status;
      if (gemm(gdn, c.dtype, st) != cudaSuccess) return HYMBA_ERR_CUDA;
    }
  }
  return HYMBA_OK;
}

hymba_status_t hymba_workspace_status(void* workspace, void* stream) {
  if (!workspace) return HYMBA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(unsigned), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return HYMBA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return HYMBA_ERR_CUDA;
  if (v != 0) {
    if (cudaMemsetAsync(workspace, 0, sizeof(unsigned), st) != cudaSuccess) return HYMBA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return HYMBA_ERR_CUDA;
    return v == HYMBA_ERR_TIMEOUT ? HYMBA_ERR_TIMEOUT : HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

hymba_status_t hymba_gemm(const void* a, const void* w, void* c, int M, int N, int K, hymba_dtype_t dtype,
                          void* workspace, size_t ws_bytes, void* stream) {
  if (!a || !w || !c || M < 1 || N < 1 || K < 1) return HYMBA_ERR_INVALID_ARG;
  if (dtype != HYMBA_BF16 && dtype != HYMBA_F32) return HYMBA_ERR_INVALID_ARG;
  if (dtype == HYMBA_BF16 && (K % 8 || N % 16)) return HYMBA_ERR_UNSUPPORTED;
  if (!workspace || ws_bytes < 256) return HYMBA_ERR_WORKSPACE;
  GemmDesc g;
  g.a = a;
  g.a_rows = M;
  g.K = K;
  g.w = w;
  g.N = N;
  g.seg[g.nseg++] = seg(0, N, c, N, 0, hy::SEG_STORE);
  g.status = static_cast<unsigned*>(workspace);
  return cuda_status(gemm(g, dtype, static_cast<cudaStream_t>(stream)));
}

hymba_status_t hymba_selective_scan(const void* x, const void* dt, const float* bc, const void* gate,
                                    const float* a_log, void* y, int y_ld, int batch, int T, int d_inner,
                                    int d_state, int a_per_state, hymba_dtype_t dtype, void* workspace,
                                    size_t ws_bytes, void* stream) {
  if (!x || !dt || !bc || !gate || !a_log || !y || batch < 1 || T < 1 || d_inner < 1 || y_ld < d_inner ||
      (a_per_state != 0 && a_per_state != 1))
    return HYMBA_ERR_INVALID_ARG;
  if (dtype != HYMBA_BF16 && dtype != HYMBA_F32) return HYMBA_ERR_INVALID_ARG;
  if (!valid_state(d_state)) return HYMBA_ERR_UNSUPPORTED;
  if (!workspace || ws_bytes < 256) return HYMBA_ERR_WORKSPACE;
  hy::ScanDesc s;
  s.x = x;
  s.dt = dt;
  s.bc = bc;
  s.gate = gate;
  s.a_log = a_log;
  s.y = y;
  s.y_ld = y_ld;
  s.batch = batch;
  s.T = T;
  s.d_inner = d_inner;
  s.d_state = d_state;
  s.bf16 = dtype == HYMBA_BF16;
  s.a_per_state = a_per_state != 0;
  s.status = static_cast<unsigned*>(workspace);
  return cuda_status(hy::launch_scan(s, static_cast<cudaStream_t>(stream)));
}

hymba_status_t hymba_attention(const void* q, const void* kv, void* out, int out_ld, int batch, int T,
                               int n_q_heads, int n_kv_heads, int head_dim, int n_meta, int window,
                               hymba_dtype_t dtype, void* workspace, size_t ws_bytes, void* stream) {
  if (!q || !kv || !out || batch < 1 || T < 1 || n_q_heads < 1 || n_kv_heads < 1 || head_dim < 1 || n_meta < 0 ||
      window < -1 || n_q_heads % n_kv_heads)
    return HYMBA_ERR_INVALID_ARG;
  if (out_ld < n_q_heads * head_dim) return HYMBA_ERR_INVALID_ARG;
  if (dtype != HYMBA_BF16 && dtype != HYMBA_F32) return HYMBA_ERR_INVALID_ARG;
  if (dtype == HYMBA_BF16 && (head_dim != 128 || out_ld % 8)) return HYMBA_ERR_UNSUPPORTED;
  if (dtype == HYMBA_F32 && head_dim > 128) return HYMBA_ERR_UNSUPPORTED;
  if (!workspace || ws_bytes < 256) return HYMBA_ERR_WORKSPACE;
  const size_t es = esize(dtype);
  const long long wkv = static_cast<long long>(n_kv_heads) * head_dim;
  hy::AttnDesc a;
  a.q = q;
  a.q_ld = static_cast<long long>(n_q_heads) * head_dim;
  a.k = kv;
  a.v = static_cast<const uint8_t*>(kv) + static_cast<size_t>(batch) * T * wkv * es;
  a.kv_ld = wkv;
  a.out = out;
  a.out_ld = out_ld;
  a.batch = batch;
  a.T = T;
  a.n_q_heads = n_q_heads;
  a.n_kv_heads = n_kv_heads;
  a.head_dim = head_dim;
  a.n_meta = n_meta;
  a.window = window;
  a.bf16 = dtype == HYMBA_BF16;
  a.status = static_cast<unsigned*>(workspace);
  return cuda_status(hy::launch_attention(a, static_cast<cudaStream_t>(stream)));
}

hymba_status_t hymba_branch_norm(void* z, const float* beta1, const float* beta2, int rows, int w_attn, int w_ssm,
                                 float eps, hymba_dtype_t dtype, void* stream) {
  if (!z || !beta1 || !beta2 || rows < 1 || w_attn < 1 || w_ssm < 1 || !(eps >= 0.f)) return HYMBA_ERR_INVALID_ARG;
  if (dtype != HYMBA_BF16 && dtype != HYMBA_F32) return HYMBA_ERR_INVALID_ARG;
  if (w_attn % 8 || w_ssm % 8) return HYMBA_ERR_UNSUPPORTED;
  return cuda_status(hy::launch_branch_norm(z, beta1, beta2, rows, w_attn, w_ssm, eps, dtype == HYMBA_BF16,
                                            static_cast<cudaStream_t>(stream)));
}

hymba_status_t hymba_rmsnorm(const void* x, void* y, int rows, int d, float eps, hymba_dtype_t dtype, void* stream) {
  if (!x || !y || rows < 1 || d < 1 || !(eps >= 0.f)) return HYMBA_ERR_INVALID_ARG;
  if (dtype != HYMBA_BF16 && dtype != HYMBA_F32) return HYMBA_ERR_INVALID_ARG;
  if (d % 8) return HYMBA_ERR_UNSUPPORTED;
  return cuda_status(hy::launch_rmsnorm(x, y, rows, d, eps, dtype == HYMBA_BF16, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
