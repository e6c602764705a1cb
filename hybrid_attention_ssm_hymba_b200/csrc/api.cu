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
#include <map>
#include <mutex>
#include <utility>

#include "hy_common.cuh"
#include "hy_kernels.h"
#include "hymba.h"

namespace hy {  // gemv.cu
bool gemv_bf16_takes(const GemmDesc& g);
cudaError_t launch_gemv_bf16(const GemmDesc& g, cudaStream_t st);
}  // namespace hy

namespace {

using hy::GemmDesc;
using hy::Seg;

inline size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
inline size_t esize(hymba_dtype_t t) { return t == HYMBA_BF16 ? 2 : 4; }

struct LayerWs {
  size_t q, kv, xs, g, dtlow, bc, dt, z, ssq, wsc, xc, total;
};

// bf16 layers fuse the branch norm into out_proj (the row-sum kernel holds a row of up
// to 6144 bf16 in one warp's registers); fp32 layers and per-group norms run a separate
// norm kernel.
bool fused_branch_norm(const hymba_cfg_t& c) {
  return c.dtype == HYMBA_BF16 && c.norm_group == 0 && c.n_q_heads * c.head_dim + c.d_inner <= 6144;
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
  // dt, or (d_state 128 with dt_proj fused into the scan, which stores no dt) the
  // blocks' shared operands, 36 KB per 32 rows (C B^T, B^T and C, fp32)
  const size_t dt_bytes = rows * c.d_inner * es, mgram = c.d_state == 128 ? (rows + 31 * c.batch) / 32 * 36864 : 0;
  w.dt = o; o = al256(o + (dt_bytes > mgram ? dt_bytes : mgram));
  w.z = o; o = al256(o + rows * (wa + c.d_inner) * es);
  // fused branch norm (bf16): per row, the sums of squares of Y_attn and Y_ssm; and
  // W_out with beta1 | beta2 folded into its columns
  const bool fused = fused_branch_norm(c);
  w.ssq = o; o = al256(o + (fused ? rows * 2 * sizeof(float) : 0));
  w.wsc = o; o = al256(o + (fused ? static_cast<size_t>(c.d_model) * (wa + c.d_inner) * es : 0));
  w.xc = o; o = al256(o + (c.conv_width > 0 ? rows * c.d_inner * es : 0));   // SiLU(conv(X_ssm))
  w.total = o;
  return w;
}

// Workspace of hymba_stack_fwd (after the 256-byte status word): the largest layer's
// workspace, the normalised block input xn (dtype) and, for bf16, its rounding remainder
// xlo and the fp32 residual stream h; K/V of the current pair; the FFN activation; for
// bf16 the transposed W_SSM and W_eff = W_x W_SSM of the current block.
struct StackWs {
  size_t layer, xn, h, kv, act, wssm_t, weff, whi, wlohi, total;
};

StackWs stack_ws(const hymba_cfg_t* cfgs, int n) {
  const hymba_cfg_t& c = cfgs[0];
  const size_t es = esize(c.dtype);
  const bool bf16 = c.dtype == HYMBA_BF16;
  const size_t rows = static_cast<size_t>(c.batch) * (c.seq_len + c.n_meta);
  const size_t d = static_cast<size_t>(c.d_model);
  size_t layer_max = 0, kvw = 0, ffn = 0, di = 0, xw = 0;
  for (int i = 0; i < n; ++i) {
    const size_t t = layer_ws(cfgs[i], 0).total;
    layer_max = t > layer_max ? t : layer_max;
    const size_t k = static_cast<size_t>(cfgs[i].n_kv_heads) * cfgs[i].head_dim;
    kvw = k > kvw ? k : kvw;
    ffn = static_cast<size_t>(cfgs[i].ffn_dim) > ffn ? cfgs[i].ffn_dim : ffn;
    di = static_cast<size_t>(cfgs[i].d_inner) > di ? cfgs[i].d_inner : di;
    const size_t x = static_cast<size_t>(cfgs[i].dt_rank) + 2 * cfgs[i].d_state;
    xw = x > xw ? x : xw;
  }
  StackWs w;
  size_t o = 0;
  w.layer = o; o = al256(o + layer_max);
  w.xn = o; o = al256(o + rows * d * es * (bf16 ? 2 : 1));   // bf16: [x_hi | x_lo] per row
  w.h = o; o = al256(o + (bf16 ? rows * d * 4 : 0));
  w.kv = o; o = al256(o + 2 * rows * kvw * es);
  w.act = o; o = al256(o + rows * ffn * es);
  w.wssm_t = o; o = al256(o + (bf16 ? d * di * 2 : 0));
  w.weff = o; o = al256(o + (bf16 ? xw * d * 4 : 0));        // W_x W_SSM, fp32
  w.whi = o; o = al256(o + (bf16 ? xw * d * 2 : 0));
  w.wlohi = o; o = al256(o + (bf16 ? xw * d * 4 : 0));       // [W_lo | W_hi]
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
  if (c->conv_width < 0 || c->conv_width > 4 || c->fusion < 0 || c->fusion > 1 || c->norm_group < 0)
    return HYMBA_ERR_INVALID_ARG;
  if (c->norm_group && ((c->norm_group != 64 && c->norm_group != 128 && c->norm_group != 256) ||
                        (c->n_q_heads * c->head_dim) % c->norm_group || c->d_inner % c->norm_group))
    return HYMBA_ERR_UNSUPPORTED;
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

// A product with a handful of rows (a generation step) streams W on the CUDA cores
// (gemv.cu); every other one runs on the tensor-core GEMM.
cudaError_t gemm(const GemmDesc& g, hymba_dtype_t t, cudaStream_t st) {
  if (t == HYMBA_BF16 && hy::gemv_bf16_takes(g)) return hy::launch_gemv_bf16(g, st);
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
  if (c.conv_width > 0 && (!w->w_conv || !w->b_conv)) return false;
  return true;
}

// The attention heads and the SSM heads of a layer are independent until the branch
// norm: the attention runs on a second stream of the library's, forked from the caller's
// stream after in_proj and joined back before the norm, so that its CTAs and the scan's
// fill the SMs together.  One second stream (with its fork and join events) per host
// thread, device and stream priority: calls from different threads never share one, and
// the attention keeps the caller stream's priority.  Calls made on several streams from
// the same thread do share it (their attention launches are ordered on it).
struct SideStream {
  cudaStream_t st = nullptr;
  cudaEvent_t forked = nullptr, done = nullptr;
};

bool side_stream(cudaStream_t caller, SideStream* out) {
  thread_local std::map<std::pair<int, int>, SideStream> cache;
  int dev = 0, prio = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaStreamGetPriority(caller, &prio) != cudaSuccess) return false;
  SideStream& e = cache[std::make_pair(dev, prio)];
  if (!e.st) {
    if (cudaStreamCreateWithPriority(&e.st, cudaStreamNonBlocking, prio) != cudaSuccess) {
      e.st = nullptr;
      return false;
    }
    if (cudaEventCreateWithFlags(&e.forked, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&e.done, cudaEventDisableTiming) != cudaSuccess) {
      cudaStreamDestroy(e.st);
      e = SideStream();
      return false;
    }
  }
  *out = e;
  return true;
}

// Joins the side stream back into the caller's stream once (at join() or on any return).
struct SideJoin {
  cudaStream_t st = nullptr;
  cudaEvent_t done = nullptr;
  cudaError_t join() {
    if (!done) return cudaSuccess;
    const cudaError_t e = cudaStreamWaitEvent(st, done, 0);
    done = nullptr;
    return e;
  }
  ~SideJoin() { join(); }
};

// Where a layer's out_proj writes: out = Z W_out^T, or out = resid + Z W_out^T (resid may
// alias out), each in the layer's dtype or in fp32 (a stack's fp32 residual stream).
// a_ld: row stride of the layer input x (plain mode; 0 = d_model).
// w_hi / w_lohi: a stacked block's x_proj straight from its input: [dt_low | B | C] =
// X_ssm W_x^T = x (W_x W_SSM)^T, evaluated as x_hi W_hi^T + [x_hi | x_lo] [W_lo | W_hi]^T with
// x_hi the bf16 normalised input, x_lo its bf16 rounding remainder (the columns of x after
// x_hi: x is [rows, 2 d] with row stride a_ld), W_hi + W_lo = W_x W_SSM to ~16 bits.
// h_out: the SSM heads' state after the last row [B, Di, N] fp32 (a prefill that a
// generation step continues); kv_rows: rows per sequence of a consumed K/V buffer (a cache).
struct LayerOut {
  void* out = nullptr;
  const void* resid = nullptr;
  bool resid_f32 = false, out_f32 = false;
  long long a_ld = 0;
  const void* w_hi = nullptr;
  const void* w_lohi = nullptr;
  float* h_out = nullptr;
  long long kv_rows = 0;
  // Meta-prefix record (hymba_meta_prefix): x holds the user rows [B, L, d] only; the meta
  // rows' K/V, SSM state and outputs come from the record instead of being recomputed.
  const uint8_t* prefix = nullptr;
};

// Layout of a meta-prefix record (offsets in bytes): the M meta rows' layer output
// [M, d] (dtype), their K then V [2, M, Hkv*dh] (dtype; none for a consuming layer) and
// the SSM state after them [Di, N] fp32.
struct PrefixLayout {
  size_t out, kv, h, total;
};
PrefixLayout prefix_layout(const hymba_cfg_t& c) {
  const size_t es = esize(c.dtype), M = static_cast<size_t>(c.n_meta);
  const size_t wkv = static_cast<size_t>(c.n_kv_heads) * c.head_dim;
  PrefixLayout p;
  size_t o = 0;
  p.out = o; o = al256(o + M * c.d_model * es);
  p.kv = o; o = al256(o + (c.kv_mode == HYMBA_KV_CONSUME ? 0 : 2 * M * wkv * es));
  p.h = o; o = al256(o + static_cast<size_t>(c.d_inner) * c.d_state * 4);
  p.total = o;
  return p;
}

// One layer.  x: meta mode when meta != nullptr, else [rows, d] holding X~.
hymba_status_t run_layer(const void* x, const void* meta, const hymba_weights_t& w, const hymba_cfg_t& c,
                         const void* kv_in, void* kv_out, const LayerOut& lo, uint8_t* ws, unsigned* status,
                         cudaStream_t st, void* const* events = nullptr) {
  void* out = lo.out;
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

  // the SSM heads' input: X_ssm, or SiLU(conv(X_ssm)) with the Mamba conv
  void* xin_ssm = c.conv_width > 0 ? static_cast<void*>(ws + L.xc) : xs;
  const float s2 = c.fusion ? -1.f : 1.f;   // difference fusion: the SSM branch subtracted
  hy::ScanDesc sd;
  sd.x = xin_ssm;
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
  sd.h_out = lo.h_out;
  const PrefixLayout PL = prefix_layout(c);
  if (lo.prefix) {   // the scan starts after the meta rows, from their state
    sd.t0 = c.n_meta;
    sd.h0 = reinterpret_cast<const float*>(lo.prefix + PL.h);
    sd.h0_bstride = 0;
  }
  // bf16 with d_state 16 (dt_rank 64) or 128 (dt_rank 8..128, a multiple of 8): dt_proj
  // runs inside the tensor-core scan (dt = softplus(dt_low W_dt^T + b_dt) per block,
  // never stored)
  {
    hy::ScanDesc f = sd;
    f.dt_low = dtlow;
    f.w_dt = w.w_dt;
    f.b_dt = w.b_dt;
    f.dt_rank = c.dt_rank;
    f.mgram = dt;   // unused as dt when fused
    // Not for a prefixed call with d_state 128: the tensor-core scan started after the meta
    // rows from a stored state gave wrong outputs in a few rows of its first block,
    // intermittently, which shows a premature read that is not yet found; such a call takes
    // dt_proj as a GEMM and the CUDA-core scan instead.
    if (!(lo.prefix && c.d_state == 128) && hy::scan_tc_fuses_dt(f)) sd = f;
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
  const long long kv_seq_rows = (c.kv_mode == HYMBA_KV_CONSUME && lo.kv_rows > 0) ? lo.kv_rows : T;
  const void* kv_v = static_cast<const uint8_t*>(kv_k) + static_cast<size_t>(c.batch) * kv_seq_rows * wkv * es;

  // 1 in_proj
  mark(0);
  GemmDesc gi;
  if (lo.prefix) {   // user rows only, written at their places in the [B, T] layout
    gi.a = x;
    gi.a_rows = static_cast<long long>(c.batch) * c.seq_len;
    gi.remap_L = c.seq_len;
    gi.remap_T = T;
    gi.remap_M = c.n_meta;
  } else if (meta) {
    gi.meta_mode = true;
    gi.x = x;
    gi.meta = meta;
    gi.batch = c.batch;
    gi.L = c.seq_len;
    gi.n_meta = c.n_meta;
  } else {
    gi.a = x;
    gi.a_rows = rows;
    gi.a_ld = lo.a_ld;
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
  if (lo.prefix && c.kv_mode != HYMBA_KV_CONSUME) {   // the meta rows' K, V into every sequence
    const size_t blk = static_cast<size_t>(c.n_meta) * wkv * es, seq = static_cast<size_t>(T) * wkv * es;
    if (hy::launch_broadcast(lo.prefix + PL.kv, blk, kvbuf, seq, c.batch, st) != cudaSuccess ||
        hy::launch_broadcast(lo.prefix + PL.kv + blk, blk, static_cast<uint8_t*>(kvbuf) + rows * wkv * es, seq,
                             c.batch, st) != cudaSuccess)
      return HYMBA_ERR_CUDA;
  }

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
  ad.kv_rows = c.kv_mode == HYMBA_KV_CONSUME ? lo.kv_rows : 0;
  ad.q_row0 = lo.prefix ? c.n_meta : 0;
  SideStream ss;
  cudaStream_t side = nullptr;
  if (!events) {
    if (!side_stream(st, &ss)) return HYMBA_ERR_CUDA;
    side = ss.st;
  }
  SideJoin joiner;
  joiner.st = st;
  if (side) {
    if (cudaEventRecord(ss.forked, st) != cudaSuccess || cudaStreamWaitEvent(side, ss.forked, 0) != cudaSuccess)
      return HYMBA_ERR_CUDA;
    const cudaError_t ea = hy::launch_attention(ad, side);
    if (cudaEventRecord(ss.done, side) != cudaSuccess) return HYMBA_ERR_CUDA;
    joiner.done = ss.done;
    if (ea != cudaSuccess) return HYMBA_ERR_CUDA;
  }

  // 2 x_proj (after the conv, when the layer has one)
  mark(1);
  if (c.conv_width > 0 && hy::launch_conv_silu(xs, w.w_conv, w.b_conv, xin_ssm, c.batch, T, di, c.conv_width,
                                               c.dtype == HYMBA_BF16, st) != cudaSuccess)
    return HYMBA_ERR_CUDA;
  GemmDesc gx;
  gx.a_rows = rows;
  gx.N = c.dt_rank + 2 * c.d_state;
  if (lo.w_hi && c.dtype == HYMBA_BF16) {   // from the layer input, compensated (see LayerOut)
    gx.a = x;
    gx.a_ld = lo.a_ld;
    gx.K = c.d_model;
    gx.w = lo.w_hi;
    gx.a2 = x;
    gx.K2 = 2 * c.d_model;
    gx.w2 = lo.w_lohi;
  } else {
    gx.a = xin_ssm;
    gx.K = di;
    gx.w = w.w_x;
  }
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
  if (e == cudaSuccess && w.d_skip)   // Mamba's D skip on the scan's output columns
    e = hy::launch_ssm_skip(static_cast<uint8_t*>(z) + wa * es, wa + di, g, xin_ssm, w.d_skip, rows, di,
                            c.dtype == HYMBA_BF16, st);
  if (joiner.join() != cudaSuccess || e != cudaSuccess) return HYMBA_ERR_CUDA;  // the norm reads all of Z

  // 6 per-branch RMSNorm and beta
  mark(5);
  if (fused_norm) {
    if ((e = hy::launch_scale_cols(w.w_out, w_out_scaled, c.d_model, wa, di, w.beta1, w.beta2, st, s2)) !=
            cudaSuccess ||
        (e = hy::launch_row_ssq(z, rows, wa, di, ssq, st, status)) != cudaSuccess)
      return HYMBA_ERR_CUDA;
  } else if (c.norm_group) {
    if ((e = hy::launch_group_norm(z, rows, wa, di, c.norm_group, w.beta1, w.beta2, s2, c.rms_eps,
                                   c.dtype == HYMBA_BF16, st)) != cudaSuccess)
      return HYMBA_ERR_CUDA;
  } else if ((e = hy::launch_branch_norm(z, w.beta1, w.beta2, rows, wa, di, c.rms_eps, c.dtype == HYMBA_BF16, st,
                                         s2)) != cudaSuccess) {
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
  if (lo.resid) {
    go.epi = hy::EPI_RESIDUAL;
    go.resid = lo.resid;
    go.resid_ld = c.d_model;
    go.out = out;
    go.out_ld = c.d_model;
    go.resid_f32 = lo.resid_f32;
    go.out_f32 = lo.out_f32;
  } else {
    go.seg[go.nseg++] = seg(0, c.d_model, out, c.d_model, f32out, hy::SEG_STORE);
  }
  go.status = status;
  if ((e = gemm(go, c.dtype, st)) != cudaSuccess) return HYMBA_ERR_CUDA;
  if (lo.prefix && hy::launch_broadcast(lo.prefix + PL.out, static_cast<size_t>(c.n_meta) * c.d_model * es, out,
                                        static_cast<size_t>(T) * c.d_model * es, c.batch, st) != cudaSuccess)
    return HYMBA_ERR_CUDA;   // the meta rows' outputs
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

// ---- generation (prefill with state, decode step)

constexpr int kMaxDecodeSplits = 256;

struct DecodeWs {
  size_t q, xs, g, dt, dtlow, bc, z, part, total;
};

DecodeWs decode_ws(const hymba_cfg_t& c) {
  const size_t es = esize(c.dtype), B = static_cast<size_t>(c.batch);
  const size_t wa = static_cast<size_t>(c.n_q_heads) * c.head_dim;
  DecodeWs w;
  size_t o = 0;
  w.q = o; o = al256(o + B * wa * es);
  w.xs = o; o = al256(o + B * c.d_inner * es);
  w.g = o; o = al256(o + B * c.d_inner * es);
  w.dt = o; o = al256(o + B * c.d_inner * es);
  w.dtlow = o; o = al256(o + B * c.dt_rank * es);
  w.bc = o; o = al256(o + B * 2 * c.d_state * 4);
  w.z = o; o = al256(o + B * (wa + c.d_inner) * es);
  w.part = o; o = al256(o + B * c.n_q_heads * kMaxDecodeSplits * (c.head_dim + 2) * 4);
  w.total = o;
  return w;
}

// the prefill runs the layer with its K/V in the workspace (own mode) and copies them into
// the cache; a consuming layer reads the producer's cache in place
hymba_cfg_t prefill_cfg(const hymba_cfg_t& c) {
  hymba_cfg_t p = c;
  if (p.kv_mode == HYMBA_KV_PRODUCE) p.kv_mode = HYMBA_KV_OWN;
  return p;
}

hymba_status_t validate_generation(const hymba_cfg_t* cfg) {
  hymba_status_t s = validate_cfg(cfg);
  if (s != HYMBA_OK) return s;
  if (cfg->conv_width > 0) return HYMBA_ERR_UNSUPPORTED;   // no convolution state is carried
  if (cfg->head_dim % 32 || cfg->n_q_heads / cfg->n_kv_heads > 8 || cfg->d_state % 8)
    return HYMBA_ERR_UNSUPPORTED;
  return HYMBA_OK;
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
  for (int i = 0; i < n_layers; ++i)
    if (validate_cfg(&cfgs[i]) != HYMBA_OK) return 0;
  return 256 + stack_ws(cfgs, n_layers).total;
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
  LayerOut lo;
  lo.out = out;
  return run_layer(x, cfg->n_meta > 0 ? meta : nullptr, *w, *cfg, kv_in, kv_out, lo,
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
  LayerOut lo;
  lo.out = out;
  return run_layer(x, cfg->n_meta > 0 ? meta : nullptr, *w, *cfg, kv_in, kv_out, lo, scratch + 256, status, st);
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

  const StackWs S = stack_ws(cfgs, n_layers);
  uint8_t* base = static_cast<uint8_t*>(workspace) + 256;
  const bool bf16 = c0.dtype == HYMBA_BF16;
  const int T = c0.seq_len + c0.n_meta;
  const long long rows = static_cast<long long>(c0.batch) * T;
  const int d = c0.d_model;
  uint8_t* lws = base + S.layer;
  void* xn = base + S.xn;   // bf16: row r = [x_hi (d) | x_lo (d)], row stride 2 d
  const long long xn_ld = bf16 ? 2LL * d : d;
  void* kv = base + S.kv;
  void* act = base + S.act;
  // the residual stream h: fp32 in the workspace (bf16), or `out` itself (fp32)
  float* h = bf16 ? reinterpret_cast<float*>(base + S.h) : static_cast<float*>(out);
  void* wssm_t = base + S.wssm_t;
  float* weff = reinterpret_cast<float*>(base + S.weff);
  void* whi = base + S.whi;
  void* wlohi = base + S.wlohi;

  cudaError_t e;
  if (bf16) {
    if ((e = hy::launch_prepend_f32(x, meta, h, c0.batch, c0.seq_len, c0.n_meta, d, st)) != cudaSuccess)
      return HYMBA_ERR_CUDA;
  } else {
    // h = [meta; x] lives in `out` and is updated in place
    const long long row_vecs = static_cast<long long>(d) * 4 / 16;
    const long long total = rows * row_vecs;
    const int blocks = static_cast<int>(total / 256 + 1 < 4096 ? total / 256 + 1 : 4096);
    if (hy::launch(prepend_kernel, dim3(blocks), dim3(256), 0, st, static_cast<const uint4*>(x),
                   static_cast<const uint4*>(meta), static_cast<uint4*>(out), row_vecs, c0.seq_len, c0.n_meta,
                   total) != cudaSuccess)
      return HYMBA_ERR_CUDA;
  }
  for (int i = 0; i < n_layers; ++i) {
    const hymba_cfg_t& c = cfgs[i];
    const bool last = i == n_layers - 1;
    LayerOut lo;
    lo.resid = h;
    lo.resid_f32 = true;
    // the last sub-block rounds h into `out` (bf16); every other one updates h in place
    const bool mixer_last = last && c.ffn_dim == 0;
    lo.out = (bf16 && mixer_last) ? out : static_cast<void*>(h);
    lo.out_f32 = !(bf16 && mixer_last);
    // x_proj straight from the block input (linear in it): not with the conv option
    const bool compensate = bf16 && c.conv_width == 0;
    lo.a_ld = xn_ld;
    if (bf16) {
      if ((e = hy::launch_prenorm_f32(h, w[i].norm1, xn, compensate ? static_cast<uint8_t*>(xn) + d * 2 : nullptr,
                                      rows, d, c.rms_eps, st, xn_ld)) != cudaSuccess)
        return HYMBA_ERR_CUDA;
    }
    if (compensate) {
      // W_eff = W_x W_SSM [R + 2N, d] in fp32, split into bf16 W_hi + W_lo
      const int wa = c.n_q_heads * c.head_dim, wkv = c.n_kv_heads * c.head_dim;
      const int ssm_row0 = wa + (c.kv_mode == HYMBA_KV_CONSUME ? 0 : 2 * wkv);
      const int xw = c.dt_rank + 2 * c.d_state;
      const uint8_t* wssm = static_cast<const uint8_t*>(w[i].w_in) + static_cast<size_t>(ssm_row0) * d * 2;
      if ((e = hy::launch_transpose_bf16(wssm, d, wssm_t, c.d_inner, d, st)) != cudaSuccess) return HYMBA_ERR_CUDA;
      GemmDesc ge;
      ge.a = w[i].w_x;
      ge.a_rows = xw;
      ge.K = c.d_inner;
      ge.w = wssm_t;
      ge.N = d;
      ge.seg[ge.nseg++] = seg(0, d, weff, d, 1, hy::SEG_STORE);
      ge.status = status;
      if (gemm(ge, c.dtype, st) != cudaSuccess) return HYMBA_ERR_CUDA;
      if ((e = hy::launch_split_hi_lo(weff, whi, wlohi, xw, d, st)) != cudaSuccess) return HYMBA_ERR_CUDA;
      lo.w_hi = whi;
      lo.w_lohi = wlohi;
    } else if (!bf16 && (e = hy::launch_prenorm_f32_out_f32(h, w[i].norm1, static_cast<float*>(xn), rows, d,
                                                            c.rms_eps, st)) != cudaSuccess) {
      return HYMBA_ERR_CUDA;
    }
    hymba_status_t s = run_layer(xn, nullptr, w[i], c, kv, kv, lo, lws, status, st);
    if (s != HYMBA_OK) return s;
    if (c.ffn_dim > 0) {
      e = bf16 ? hy::launch_prenorm_f32(h, w[i].norm2, xn, nullptr, rows, d, c.rms_eps, st, xn_ld)
               : hy::launch_prenorm_f32_out_f32(h, w[i].norm2, static_cast<float*>(xn), rows, d, c.rms_eps, st);
      if (e != cudaSuccess) return HYMBA_ERR_CUDA;
      GemmDesc gu;
      gu.a = xn;
      gu.a_ld = xn_ld;
      gu.a_rows = rows;
      gu.K = d;
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
      gdn.N = d;
      gdn.epi = hy::EPI_RESIDUAL;
      gdn.resid = h;
      gdn.resid_ld = d;
      gdn.resid_f32 = true;
      gdn.out = (bf16 && last) ? out : static_cast<void*>(h);
      gdn.out_f32 = !(bf16 && last);
      gdn.out_ld = d;
      gdn.status = status;
      if (gemm(gdn, c.dtype, st) != cudaSuccess) return HYMBA_ERR_CUDA;
    }
  }
  return HYMBA_OK;
}

// ---- generation: prefill that keeps the K/V cache and the SSM state, then one token per step

size_t hymba_decode_workspace_size(const hymba_cfg_t* cfg) {
  if (validate_generation(cfg) != HYMBA_OK) return 0;
  const hymba_cfg_t p = prefill_cfg(*cfg);
  const size_t a = layer_ws(p, 0).total, b = decode_ws(*cfg).total;
  return 256 + (a > b ? a : b);
}

hymba_status_t hymba_layer_prefill(const void* x, const void* meta, const hymba_weights_t* w, const hymba_cfg_t* cfg,
                                   void* kv_cache, int cache_rows, float* ssm_state, void* out, void* workspace,
                                   size_t ws_bytes, void* stream) {
  hymba_status_t s = validate_generation(cfg);
  if (s != HYMBA_OK) return s;
  const int T = cfg->seq_len + cfg->n_meta;
  if (!x || !out || !kv_cache || !ssm_state || !weights_ok(w, *cfg, false) || cache_rows < T)
    return HYMBA_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < hymba_decode_workspace_size(cfg)) return HYMBA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255) return HYMBA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned* status = static_cast<unsigned*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(unsigned), st) != cudaSuccess) return HYMBA_ERR_CUDA;
  const hymba_cfg_t p = prefill_cfg(*cfg);
  uint8_t* ws = static_cast<uint8_t*>(workspace) + 256;
  LayerOut lo;
  lo.out = out;
  lo.h_out = ssm_state;
  lo.kv_rows = cache_rows;
  s = run_layer(x, cfg->n_meta > 0 ? meta : nullptr, *w, p, cfg->kv_mode == HYMBA_KV_CONSUME ? kv_cache : nullptr,
                nullptr, lo, ws, status, st);
  if (s != HYMBA_OK || cfg->kv_mode == HYMBA_KV_CONSUME) return s;
  // K, V [2][B*T][wkv] in the workspace -> the cache [2][B][cache_rows][wkv]
  const size_t es = esize(cfg->dtype), wkv = static_cast<size_t>(cfg->n_kv_heads) * cfg->head_dim;
  const LayerWs L = layer_ws(p, 0);
  if (cudaMemcpy2DAsync(kv_cache, static_cast<size_t>(cache_rows) * wkv * es, ws + L.kv, T * wkv * es,
                        T * wkv * es, 2 * static_cast<size_t>(cfg->batch), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return HYMBA_ERR_CUDA;
  return HYMBA_OK;
}

hymba_status_t hymba_layer_decode(const void* x_t, const hymba_weights_t* w, const hymba_cfg_t* cfg, void* kv_cache,
                                  int cache_rows, int pos, float* ssm_state, void* out_t, void* workspace,
                                  size_t ws_bytes, void* stream) {
  hymba_status_t s = validate_generation(cfg);
  if (s != HYMBA_OK) return s;
  const hymba_cfg_t& c = *cfg;
  if (!x_t || !out_t || !kv_cache || !ssm_state || !weights_ok(w, c, false) || pos < 0 || pos >= cache_rows)
    return HYMBA_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < hymba_decode_workspace_size(cfg)) return HYMBA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255) return HYMBA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned* status = static_cast<unsigned*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(unsigned), st) != cudaSuccess) return HYMBA_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace) + 256;
  const DecodeWs D = decode_ws(c);
  const size_t es = esize(c.dtype);
  const int wa = c.n_q_heads * c.head_dim, wkv = c.n_kv_heads * c.head_dim, di = c.d_inner, B = c.batch;
  const long long cache_ld = static_cast<long long>(cache_rows) * wkv;   // elements between sequences
  uint8_t* kc = static_cast<uint8_t*>(kv_cache);
  uint8_t* vc = kc + static_cast<size_t>(B) * cache_ld * es;
  void* q = ws + D.q;
  void* xs = ws + D.xs;
  void* g = ws + D.g;
  void* dt = ws + D.dt;
  void* dtlow = ws + D.dtlow;
  float* bc = reinterpret_cast<float*>(ws + D.bc);
  void* z = ws + D.z;
  // in_proj of the new rows; K, V go straight into the cache at row pos
  GemmDesc gi;
  gi.a = x_t;
  gi.a_rows = B;
  gi.K = c.d_model;
  gi.w = w->w_in;
  int col = 0;
  gi.seg[gi.nseg++] = seg(col, col + wa, q, wa, 0, hy::SEG_STORE);
  col += wa;
  if (c.kv_mode != HYMBA_KV_CONSUME) {
    gi.seg[gi.nseg++] = seg(col, col + wkv, kc + static_cast<size_t>(pos) * wkv * es, cache_ld, 0, hy::SEG_STORE);
    col += wkv;
    gi.seg[gi.nseg++] = seg(col, col + wkv, vc + static_cast<size_t>(pos) * wkv * es, cache_ld, 0, hy::SEG_STORE);
    col += wkv;
  }
  gi.seg[gi.nseg++] = seg(col, col + di, xs, di, 0, hy::SEG_STORE);
  col += di;
  gi.seg[gi.nseg++] = seg(col, col + di, g, di, 0, hy::SEG_SILU);
  col += di;
  gi.N = col;
  gi.status = status;
  if (gemm(gi, c.dtype, st) != cudaSuccess) return HYMBA_ERR_CUDA;
  GemmDesc gx;
  gx.a = xs;
  gx.a_rows = B;
  gx.K = di;
  gx.w = w->w_x;
  gx.N = c.dt_rank + 2 * c.d_state;
  gx.seg[gx.nseg++] = seg(0, c.dt_rank, dtlow, c.dt_rank, 0, hy::SEG_STORE);
  gx.seg[gx.nseg++] = seg(c.dt_rank, gx.N, bc, 2 * c.d_state, 1, hy::SEG_STORE);
  gx.status = status;
  if (gemm(gx, c.dtype, st) != cudaSuccess) return HYMBA_ERR_CUDA;
  GemmDesc gd;
  gd.a = dtlow;
  gd.a_rows = B;
  gd.K = c.dt_rank;
  gd.w = w->w_dt;
  gd.N = di;
  gd.seg[gd.nseg++] = seg(0, di, dt, di, 0, hy::SEG_SOFTPLUS_BIAS, w->b_dt);
  gd.status = status;
  if (gemm(gd, c.dtype, st) != cudaSuccess) return HYMBA_ERR_CUDA;
  // the token's query against the cached rows it sees
  hy::DecodeAttnDesc ad;
  ad.q = q;
  ad.k = kc;
  ad.v = vc;
  ad.cap = cache_rows;
  ad.kv_ld = wkv;
  ad.out = z;
  ad.out_ld = wa + di;
  ad.part = reinterpret_cast<float*>(ws + D.part);
  ad.max_splits = kMaxDecodeSplits;
  ad.batch = B;
  ad.n_q_heads = c.n_q_heads;
  ad.n_kv_heads = c.n_kv_heads;
  ad.head_dim = c.head_dim;
  ad.pos = pos;
  ad.n_meta = c.n_meta;
  ad.window = c.window;
  ad.bf16 = c.dtype == HYMBA_BF16;
  if (hy::launch_attention_decode(ad, st) != cudaSuccess) return HYMBA_ERR_CUDA;
  // one step of every SSM channel from the carried state
  hy::ScanStepDesc sd;
  sd.x = xs;
  sd.dt = dt;
  sd.bc = bc;
  sd.gate = g;
  sd.a_log = w->a_log;
  sd.a_per_state = c.a_per_state != 0;
  sd.h = ssm_state;
  sd.y = static_cast<uint8_t*>(z) + wa * es;
  sd.y_ld = wa + di;
  sd.batch = B;
  sd.d_inner = di;
  sd.d_state = c.d_state;
  sd.bf16 = c.dtype == HYMBA_BF16;
  sd.d_skip = w->d_skip;
  if (hy::launch_scan_step(sd, st) != cudaSuccess) return HYMBA_ERR_CUDA;
  const float s2 = c.fusion ? -1.f : 1.f;
  const cudaError_t en = c.norm_group ? hy::launch_group_norm(z, B, wa, di, c.norm_group, w->beta1, w->beta2, s2,
                                                              c.rms_eps, c.dtype == HYMBA_BF16, st)
                                      : hy::launch_branch_norm(z, w->beta1, w->beta2, B, wa, di, c.rms_eps,
                                                               c.dtype == HYMBA_BF16, st, s2);
  if (en != cudaSuccess) return HYMBA_ERR_CUDA;
  GemmDesc go;
  go.a = z;
  go.a_rows = B;
  go.K = wa + di;
  go.w = w->w_out;
  go.N = c.d_model;
  go.seg[go.nseg++] = seg(0, c.d_model, out_t, c.d_model, 0, hy::SEG_STORE);
  go.status = status;
  return gemm(go, c.dtype, st) == cudaSuccess ? HYMBA_OK : HYMBA_ERR_CUDA;
}

// ---- meta-prefix precompute: the meta rows once per weight set, then only the user rows

size_t hymba_meta_prefix_size(const hymba_cfg_t* cfg) {
  if (validate_cfg(cfg) != HYMBA_OK || cfg->n_meta < 1) return 0;
  return prefix_layout(*cfg).total;
}

hymba_status_t hymba_meta_prefix(const void* meta_in, const hymba_weights_t* w, const hymba_cfg_t* cfg,
                                 const void* kv_prefix_in, void* prefix, void* workspace, size_t ws_bytes,
                                 void* stream) {
  hymba_status_t s = validate_cfg(cfg);
  if (s != HYMBA_OK) return s;
  if (cfg->conv_width > 0) return HYMBA_ERR_UNSUPPORTED;   // the conv would need the meta rows' X_ssm
  if (cfg->n_meta < 1 || !meta_in || !prefix || !weights_ok(w, *cfg, false)) return HYMBA_ERR_INVALID_ARG;
  if (cfg->kv_mode == HYMBA_KV_CONSUME && !kv_prefix_in) return HYMBA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(prefix) & 255) return HYMBA_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < hymba_workspace_size(cfg)) return HYMBA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255) return HYMBA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned* status = static_cast<unsigned*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(unsigned), st) != cudaSuccess) return HYMBA_ERR_CUDA;
  // The meta rows alone, as one sequence of M rows: every meta row sees every meta row
  // before it whatever the window (all are meta tokens), so the prefix runs as global
  // causal attention; a layer with its own K/V writes them into the record.
  hymba_cfg_t p = *cfg;
  p.batch = 1;
  p.seq_len = cfg->n_meta;
  p.n_meta = 0;
  p.window = -1;
  if (p.kv_mode == HYMBA_KV_OWN) p.kv_mode = HYMBA_KV_PRODUCE;
  const PrefixLayout PL = prefix_layout(*cfg);
  uint8_t* rec = static_cast<uint8_t*>(prefix);
  LayerOut lo;
  lo.out = rec + PL.out;
  lo.h_out = reinterpret_cast<float*>(rec + PL.h);
  lo.kv_rows = cfg->n_meta;
  // a consuming layer's meta rows read the producer's meta K/V from the producer's record
  hymba_cfg_t producer = *cfg;
  producer.kv_mode = HYMBA_KV_PRODUCE;
  const void* kv_in = cfg->kv_mode == HYMBA_KV_CONSUME
                          ? static_cast<const uint8_t*>(kv_prefix_in) + prefix_layout(producer).kv
                          : nullptr;
  return run_layer(meta_in, nullptr, *w, p, kv_in, cfg->kv_mode == HYMBA_KV_CONSUME ? nullptr : rec + PL.kv, lo,
                   static_cast<uint8_t*>(workspace) + 256, status, st);
}

hymba_status_t hymba_layer_fwd_prefixed(const void* x, const void* prefix, const hymba_weights_t* w,
                                        const hymba_cfg_t* cfg, const void* kv_in, void* kv_out, void* out,
                                        void* workspace, size_t ws_bytes, void* stream) {
  hymba_status_t s = validate_cfg(cfg);
  if (s != HYMBA_OK) return s;
  if (cfg->conv_width > 0) return HYMBA_ERR_UNSUPPORTED;
  if (cfg->n_meta < 1 || !x || !prefix || !out || !weights_ok(w, *cfg, false)) return HYMBA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(prefix) & 255) return HYMBA_ERR_INVALID_ARG;
  if (cfg->kv_mode == HYMBA_KV_CONSUME && !kv_in) return HYMBA_ERR_INVALID_ARG;
  if (cfg->kv_mode == HYMBA_KV_PRODUCE && !kv_out) return HYMBA_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < hymba_workspace_size(cfg)) return HYMBA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255) return HYMBA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned* status = static_cast<unsigned*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(unsigned), st) != cudaSuccess) return HYMBA_ERR_CUDA;
  LayerOut lo;
  lo.out = out;
  lo.prefix = static_cast<const uint8_t*>(prefix);
  return run_layer(x, nullptr, *w, *cfg, kv_in, kv_out, lo, static_cast<uint8_t*>(workspace) + 256, status, st);
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

size_t hymba_selective_scan_dtproj_workspace_size(int batch, int T, int d_inner, int d_state, int dt_rank,
                                                  hymba_dtype_t dtype) {
  if (batch < 1 || T < 1 || d_inner < 1 || dt_rank < 1) return 0;
  hy::ScanDesc f;
  f.x = f.gate = f.dt_low = f.w_dt = reinterpret_cast<const void*>(256);
  f.y = reinterpret_cast<void*>(256);
  f.bc = reinterpret_cast<const float*>(256);
  f.b_dt = reinterpret_cast<const float*>(256);
  f.y_ld = d_inner;
  f.d_inner = d_inner;
  f.d_state = d_state;
  f.dt_rank = dt_rank;
  f.bf16 = dtype == HYMBA_BF16;
  f.batch = batch;
  f.T = T;
  if (hy::scan_tc_fuses_dt(f)) return 256 + (hy::scan_mgram_bytes(f) + 255) / 256 * 256;
  const size_t es = dtype == HYMBA_BF16 ? 2 : 4;
  return 256 + (static_cast<size_t>(batch) * T * d_inner * es + 255) / 256 * 256;
}

hymba_status_t hymba_selective_scan_dtproj(const void* x, const void* dt_low, const void* w_dt, const float* b_dt,
                                           int dt_rank, const float* bc, const void* gate, const float* a_log,
                                           void* y, int y_ld, int batch, int T, int d_inner, int d_state,
                                           hymba_dtype_t dtype, void* workspace, size_t ws_bytes, void* stream) {
  if (!x || !dt_low || !w_dt || !b_dt || !bc || !gate || !a_log || !y || batch < 1 || T < 1 || d_inner < 1 ||
      dt_rank < 1 || y_ld < d_inner)
    return HYMBA_ERR_INVALID_ARG;
  if (dtype != HYMBA_BF16 && dtype != HYMBA_F32) return HYMBA_ERR_INVALID_ARG;
  if (!valid_state(d_state)) return HYMBA_ERR_UNSUPPORTED;
  const size_t need = hymba_selective_scan_dtproj_workspace_size(batch, T, d_inner, d_state, dt_rank, dtype);
  if (!workspace || ws_bytes < need) return HYMBA_ERR_WORKSPACE;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  hy::ScanDesc s;
  s.x = x;
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
  s.status = static_cast<unsigned*>(workspace);
  hy::ScanDesc f = s;
  f.dt = ws;  // unread when fused
  f.dt_low = dt_low;
  f.w_dt = w_dt;
  f.b_dt = b_dt;
  f.dt_rank = dt_rank;
  f.mgram = ws + 256;
  if (hy::scan_tc_fuses_dt(f)) return cuda_status(hy::launch_scan(f, st));
  // otherwise dt = softplus(dt_low W_dt^T + b_dt) through the GEMM into the workspace first
  void* dt = ws + 256;
  GemmDesc gd;
  gd.a = dt_low;
  gd.a_rows = static_cast<long long>(batch) * T;
  gd.K = dt_rank;
  gd.w = w_dt;
  gd.N = d_inner;
  gd.seg[gd.nseg++] = seg(0, d_inner, dt, d_inner, 0, hy::SEG_SOFTPLUS_BIAS, b_dt);
  gd.status = s.status;
  cudaError_t e = gemm(gd, dtype, st);
  if (e != cudaSuccess) return HYMBA_ERR_CUDA;
  s.dt = dt;
  return cuda_status(hy::launch_scan(s, st));
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
