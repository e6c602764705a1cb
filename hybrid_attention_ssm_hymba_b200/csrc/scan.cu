// scan.cu -- chunked selective scan fused with the output gate, for the SSM heads of
// the hybrid-head layer (blog.outta.ai Hymba review, "Design formulation": the
// mixing matrix alpha_ij = C_i (prod_{k=j+1..i} exp(A dt_k)) B_j dt_j and
// Y_ssm = G . alpha(A, B, C, dt) W_SSM X~).  The same output is computed here by
// the recurrence h_t = exp(A dt_t) h_{t-1} + dt_t B_t x_t, y_t = C_t . h_t.
//
// Work decomposition: a CTA owns CPW channels of one sequence for all T steps.
// Its NWT warps split T into NWT contiguous chunks.  Each thread holds NS of the
// N state components of one channel in registers (TPC threads per channel).
//   pass 1  every warp scans its chunk from h = 0 and keeps the end state and the
//           chunk's total log-decay sum_t A dt_t;
//   combine through shared memory: the state entering chunk w is
//           h_in(w) = sum_{k<w} exp(sum_{k<m<w} logdecay_m) hend_k, evaluated as the
//           sequential product chain, in fp32;
//   pass 2  every warp rescans its chunk from h_in(w) and emits y_t = gate_t (C_t . h_t),
//           reducing the TPC partial dot products with warp shuffles.
// The state is fp32 throughout (updated two components per instruction with the
// sm_100 packed fp32x2 FMA); dt, x and gate are read in the layer's dtype; exp(A dt)
// uses the SFU's ex2.
#include "hy_common.cuh"
#include "hy_kernels.h"

namespace hy {
namespace {

struct ScanParams {
  const void* x;
  const void* dt;
  const float* bc;
  const void* gate;
  const float* a_log;
  void* y;
  long long y_ld;
  int T, Di, N;
};

template <typename TI, int NS, int TPC, int NWT>
__global__ void __launch_bounds__(32 * NWT) scan_kernel(const ScanParams p) {
  constexpr int CPW = 32 / TPC;  // channels per warp (= per CTA)
  constexpr int N = NS * TPC;
  constexpr int NP = NS / 2;     // state pairs per thread (packed fp32x2 updates)
  constexpr int U = 4;           // time steps per unrolled group (loads issued up front)
  __shared__ float s_hend[NWT * CPW * N];
  __shared__ float s_logdec[NWT * CPW];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ch = lane / TPC, slice = lane % TPC;
  const int c = blockIdx.x * CPW + ch;
  const int b = blockIdx.y;
  const bool valid = c < p.Di;
  const int cc = valid ? c : 0;
  const int Lc = (p.T + NWT - 1) / NWT;
  const int t0 = min(p.T, warp * Lc), t1 = min(p.T, t0 + Lc);
  const int n0 = slice * NS;
  const long long row0 = static_cast<long long>(b) * p.T + t0;

  // A = -exp(A_log) in units of log2, so that exp(A dt) = exp2(A2 dt)
  const float A2 = -expf(p.a_log[cc]) * 1.4426950408889634f;

  float2 h[NP];
#pragma unroll
  for (int i = 0; i < NP; ++i) h[i] = make_float2(0.f, 0.f);
  float logdec = 0.f;

  // ---------------- pass 1: local scan from h = 0 (end state and total log-decay only)
  {
    const TI* xp = static_cast<const TI*>(p.x) + row0 * p.Di + cc;
    const TI* dp = static_cast<const TI*>(p.dt) + row0 * p.Di + cc;
    const float* bp = p.bc + row0 * 2 * N + n0;
    int t = t0;
    for (; t + U <= t1; t += U) {
      float dv[U], xv[U];
#pragma unroll
      for (int k = 0; k < U; ++k) {
        dv[k] = to_f<TI>(dp[k * p.Di]);
        xv[k] = to_f<TI>(xp[k * p.Di]);
      }
#pragma unroll
      for (int k = 0; k < U; ++k) {
        const float a = ex2_approx(A2 * dv[k]);
        const float u = dv[k] * xv[k];
        logdec = fmaf(A2, dv[k], logdec);
        const float2 a2 = make_float2(a, a), u2 = make_float2(u, u);
        const float4* B4 = reinterpret_cast<const float4*>(bp + k * 2 * N);
#pragma unroll
        for (int j = 0; j < NS / 4; ++j) {
          const float4 bb = __ldg(B4 + j);
          h[2 * j] = __ffma2_rn(a2, h[2 * j], __fmul2_rn(u2, make_float2(bb.x, bb.y)));
          h[2 * j + 1] = __ffma2_rn(a2, h[2 * j + 1], __fmul2_rn(u2, make_float2(bb.z, bb.w)));
        }
      }
      xp += U * p.Di;
      dp += U * p.Di;
      bp += U * 2 * N;
    }
    for (; t < t1; ++t) {
      const float d = to_f<TI>(*dp), xv = to_f<TI>(*xp);
      const float a = ex2_approx(A2 * d);
      const float u = d * xv;
      logdec = fmaf(A2, d, logdec);
      const float2 a2 = make_float2(a, a), u2 = make_float2(u, u);
      const float4* B4 = reinterpret_cast<const float4*>(bp);
#pragma unroll
      for (int j = 0; j < NS / 4; ++j) {
        const float4 bb = __ldg(B4 + j);
        h[2 * j] = __ffma2_rn(a2, h[2 * j], __fmul2_rn(u2, make_float2(bb.x, bb.y)));
        h[2 * j + 1] = __ffma2_rn(a2, h[2 * j + 1], __fmul2_rn(u2, make_float2(bb.z, bb.w)));
      }
      xp += p.Di;
      dp += p.Di;
      bp += 2 * N;
    }
  }
  float* my_hend = s_hend + (warp * CPW + ch) * N + n0;
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    my_hend[2 * i] = h[i].x;
    my_hend[2 * i + 1] = h[i].y;
  }
  if (slice == 0) s_logdec[warp * CPW + ch] = logdec;
  __syncthreads();

  // ---------------- combine: state entering this warp's chunk
#pragma unroll
  for (int i = 0; i < NP; ++i) h[i] = make_float2(0.f, 0.f);
  for (int k = 0; k < warp; ++k) {
    const float dec = ex2_approx(s_logdec[k * CPW + ch]);
    const float2 dec2 = make_float2(dec, dec);
    const float2* hk = reinterpret_cast<const float2*>(s_hend + (k * CPW + ch) * N + n0);
#pragma unroll
    for (int i = 0; i < NP; ++i) h[i] = __ffma2_rn(dec2, h[i], hk[i]);
  }

  // ---------------- pass 2: rescan with the carried state, emit gated output
  {
    const TI* xp = static_cast<const TI*>(p.x) + row0 * p.Di + cc;
    const TI* dp = static_cast<const TI*>(p.dt) + row0 * p.Di + cc;
    const TI* gp = static_cast<const TI*>(p.gate) + row0 * p.Di + cc;
    const float* bp = p.bc + row0 * 2 * N + n0;
    TI* yp = static_cast<TI*>(p.y) + row0 * p.y_ld + cc;
    const bool writer = valid && slice == 0;
    auto step = [&](float d, float xv, float g, const float* brow, TI* yout) {
      const float a = ex2_approx(A2 * d);
      const float u = d * xv;
      const float2 a2 = make_float2(a, a), u2 = make_float2(u, u);
      const float4* B4 = reinterpret_cast<const float4*>(brow);
      const float4* C4 = reinterpret_cast<const float4*>(brow + N);
      float2 y2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int j = 0; j < NS / 4; ++j) {
        const float4 bb = __ldg(B4 + j);
        const float4 cv = __ldg(C4 + j);
        h[2 * j] = __ffma2_rn(a2, h[2 * j], __fmul2_rn(u2, make_float2(bb.x, bb.y)));
        h[2 * j + 1] = __ffma2_rn(a2, h[2 * j + 1], __fmul2_rn(u2, make_float2(bb.z, bb.w)));
        y2 = __ffma2_rn(make_float2(cv.x, cv.y), h[2 * j], y2);
        y2 = __ffma2_rn(make_float2(cv.z, cv.w), h[2 * j + 1], y2);
      }
      float yv = y2.x + y2.y;
#pragma unroll
      for (int off = 1; off < TPC; off <<= 1) yv += __shfl_xor_sync(0xffffffffu, yv, off);
      if (writer) *yout = from_f<TI>(g * yv);
    };
    int t = t0;
    for (; t + U <= t1; t += U) {
      float dv[U], xv[U], gv[U];
#pragma unroll
      for (int k = 0; k < U; ++k) {
        dv[k] = to_f<TI>(dp[k * p.Di]);
        xv[k] = to_f<TI>(xp[k * p.Di]);
        gv[k] = to_f<TI>(gp[k * p.Di]);
      }
#pragma unroll
      for (int k = 0; k < U; ++k) step(dv[k], xv[k], gv[k], bp + k * 2 * N, yp + k * p.y_ld);
      xp += U * p.Di;
      dp += U * p.Di;
      gp += U * p.Di;
      bp += U * 2 * N;
      yp += U * p.y_ld;
    }
    for (; t < t1; ++t) {
      step(to_f<TI>(*dp), to_f<TI>(*xp), to_f<TI>(*gp), bp, yp);
      xp += p.Di;
      dp += p.Di;
      gp += p.Di;
      bp += 2 * N;
      yp += p.y_ld;
    }
  }
}

// ---------------------------------------------------------------------------------
// Single-pass TMA-staged scan (the main path).
//
// Each channel is scanned once, sequentially over all T steps (the critical path is
// T short steps; parallelism comes from channels x state slices).  A channel's N
// state components are split over TPC lanes (NS each, packed fp32x2 updates) and
// y = C . h is reduced with shuffles.  A CTA of NWARP warps (CPB channels) shares one
// STAGES-deep ring of ROWS-step TMA tiles -- x, dt, gate for its channels and the
// full B|C rows -- filled by one thread and released by the warps through an
// mbarrier; y goes out through a per-warp smem tile and a TMA store.  Tensor maps
// are 3-D ([batch][T][cols]), so no tile reads or writes across a sequence end.
//
// Scaled state: with P_t = prod exp(A dt_s) since the last rescale and g = h / P,
// g_t = g_{t-1} + (dt_t x_t / P_t) B_t and y_t = P_t (C_t . g_t).  P is kept as its
// log2 (cl) and folded back into g (g <- P g) at every tile start; when no lane's
// decay over the tile passes 2^-60 (checked warp-uniformly) the tile runs the
// unrolled fast path, otherwise the per-step path that folds on demand and restarts
// the state after a single step decaying by more than 2^-60.
template <int NP>
struct ScaledState {
  float2 g[NP];
  float cl;  // log2 of the scale P
  HY_DEV void zero() {
#pragma unroll
    for (int i = 0; i < NP; ++i) g[i] = make_float2(0.f, 0.f);
    cl = 0.f;
  }
  HY_DEV void fold() {
    const float P = ex2_approx(cl);
    const float2 P2 = make_float2(P, P);
#pragma unroll
    for (int i = 0; i < NP; ++i) g[i] = __fmul2_rn(g[i], P2);
    cl = 0.f;
  }
  // advance the scale by one step of log2-decay l2a; returns 1 / P_t
  HY_DEV float advance(float l2a) {
    float c = cl + l2a;
    if (c < -60.f) {  // rare: fold the scale into g
      fold();
      if (l2a < -60.f) {
#pragma unroll
        for (int i = 0; i < NP; ++i) g[i] = make_float2(0.f, 0.f);
        c = 0.f;
      } else {
        c = l2a;
      }
    }
    cl = c;
    return ex2_approx(-c);
  }
};

template <typename TI, int NS, int TPC>
struct V5Cfg {
  static constexpr int N = NS * TPC;
  static constexpr int NWARP = 4;
  static constexpr int CPW = 32 / TPC;        // channels per warp
  static constexpr int CPB = NWARP * CPW;     // channels per CTA
  static constexpr int ROWS = N <= 32 ? 16 : 8;  // steps per tile (B|C rows grow with N)
  static constexpr int STAGES = 4;
  static constexpr int XB = ROWS * CPB * (int)sizeof(TI);  // one x / dt / gate tile
  static constexpr int BCB = ROWS * 2 * N * 4;              // one B|C tile
  static constexpr int STAGE_B = 3 * XB + BCB;
  static constexpr int YB = ROWS * CPW * (int)sizeof(TI);   // one warp's y tile
  static constexpr int SMEM = STAGES * STAGE_B + NWARP * 2 * YB + 2 * STAGES * 8 + 16 + 128;
};

template <typename TI, int NS, int TPC>
__global__ void __launch_bounds__(128) scan_v5_kernel(const __grid_constant__ CUtensorMap tmX,
                                                      const __grid_constant__ CUtensorMap tmDT,
                                                      const __grid_constant__ CUtensorMap tmG,
                                                      const __grid_constant__ CUtensorMap tmBC,
                                                      const __grid_constant__ CUtensorMap tmY, const ScanParams p,
                                                      unsigned* status) {
  using C = V5Cfg<TI, NS, TPC>;
  constexpr int N = C::N;
  constexpr int NP = NS / 2;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ybuf = smem + C::STAGES * C::STAGE_B;  // [NWARP][2][ROWS][CPW]
  uint64_t* full = reinterpret_cast<uint64_t*>(ybuf + C::NWARP * 2 * C::YB);
  uint64_t* empty = full + C::STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + C::STAGES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chw = lane / TPC, slice = lane % TPC;  // channel within the warp, state slice
  const int cl_cta = warp * C::CPW + chw;          // channel within the CTA
  const int c = blockIdx.x * C::CPB + cl_cta;
  const int b = blockIdx.y;
  const int n0 = slice * NS;
  const int n_tiles = (p.T + C::ROWS - 1) / C::ROWS;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::NWARP);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const float A2 = c < p.Di ? -expf(p.a_log[c]) * 1.4426950408889634f : 0.f;
  const bool producer = threadIdx.x == 0;
  uint32_t issued = 0;
  auto issue = [&](int k) {  // tile k -> slot k % STAGES (tiles are issued in order)
    const int slot = k % C::STAGES;
    if (k >= C::STAGES && !mbar_wait(&empty[slot], ((k / C::STAGES) & 1) ^ 1u, status, abort_flag)) return false;
    uint8_t* st = smem + slot * C::STAGE_B;
    mbar_arrive_expect_tx(&full[slot], C::STAGE_B);
    const int col = blockIdx.x * C::CPB, t = k * C::ROWS;
    tma_load_3d(st, &tmX, &full[slot], col, t, b);
    tma_load_3d(st + C::XB, &tmDT, &full[slot], col, t, b);
    tma_load_3d(st + 2 * C::XB, &tmG, &full[slot], col, t, b);
    tma_load_3d(st + 3 * C::XB, &tmBC, &full[slot], 0, t, b);
    ++issued;
    return true;
  };
  bool ok = true;
  if (producer)
    for (int k = 0; ok && k < C::STAGES - 1 && k < n_tiles; ++k) ok = issue(k);

  ScaledState<NP> st;
  st.zero();
  uint8_t* my_y = ybuf + warp * 2 * C::YB;
  const size_t es = sizeof(TI);
  int k = 0;
  for (; k < n_tiles; ++k) {
    if (producer && ok && k + C::STAGES - 1 < n_tiles) ok = issue(k + C::STAGES - 1);
    const int slot = k % C::STAGES;
    if (!__all_sync(0xffffffffu, mbar_wait(&full[slot], (k / C::STAGES) & 1, status, abort_flag))) {
      ok = false;
      break;
    }
    const uint8_t* tile = smem + slot * C::STAGE_B;
    const uint8_t* tx = tile + cl_cta * es;
    const uint8_t* td = tile + C::XB + cl_cta * es;
    const uint8_t* tg = tile + 2 * C::XB + cl_cta * es;
    const float* tbc = reinterpret_cast<const float*>(tile + 3 * C::XB) + n0;
    const int rows = min(C::ROWS, p.T - k * C::ROWS);
    // y tile of this warp (double-buffered; the TMA store of tile k-2 must have read it)
    TI* yt = reinterpret_cast<TI*>(my_y + (k & 1) * C::YB);
    if (lane == 0) bulk_wait_read1();
    __syncwarp();

    st.fold();
    bool fast = rows == C::ROWS;
    if (fast) {
      float cum = 0.f;
#pragma unroll
      for (int r = 0; r < C::ROWS; ++r) cum = fmaf(A2, to_f<TI>(*reinterpret_cast<const TI*>(td + r * C::CPB * es)), cum);
      fast = cum >= -60.f;
    }
    if (__all_sync(0xffffffffu, fast)) {
#pragma unroll
      for (int r0 = 0; r0 < C::ROWS; r0 += 4) {  // four steps: scales first (independent SFU ops), then the chain
        float v[4], P[4], gt[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int r = r0 + q;
          const float d = to_f<TI>(*reinterpret_cast<const TI*>(td + r * C::CPB * es));
          const float xv = to_f<TI>(*reinterpret_cast<const TI*>(tx + r * C::CPB * es));
          gt[q] = to_f<TI>(*reinterpret_cast<const TI*>(tg + r * C::CPB * es));
          st.cl = fmaf(A2, d, st.cl);
          v[q] = d * xv * ex2_approx(-st.cl);
          P[q] = ex2_approx(st.cl);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int r = r0 + q;
          const float4* B4 = reinterpret_cast<const float4*>(tbc + r * 2 * N);
          const float4* C4 = reinterpret_cast<const float4*>(tbc + r * 2 * N + N);
          const float2 v2 = make_float2(v[q], v[q]);
          float2 ya = make_float2(0.f, 0.f), yb = make_float2(0.f, 0.f);
#pragma unroll
          for (int j = 0; j < NS / 4; ++j) {
            const float4 bb = B4[j], cv = C4[j];
            st.g[2 * j] = __ffma2_rn(v2, make_float2(bb.x, bb.y), st.g[2 * j]);
            st.g[2 * j + 1] = __ffma2_rn(v2, make_float2(bb.z, bb.w), st.g[2 * j + 1]);
            ya = __ffma2_rn(make_float2(cv.x, cv.y), st.g[2 * j], ya);
            yb = __ffma2_rn(make_float2(cv.z, cv.w), st.g[2 * j + 1], yb);
          }
          float y = (ya.x + ya.y) + (yb.x + yb.y);
#pragma unroll
          for (int off = 1; off < TPC; off <<= 1) y += __shfl_xor_sync(0xffffffffu, y, off);
          if (slice == 0) yt[r * C::CPW + chw] = from_f<TI>(gt[q] * P[q] * y);
        }
      }
    } else {
      for (int r = 0; r < rows; ++r) {
        const float d = to_f<TI>(*reinterpret_cast<const TI*>(td + r * C::CPB * es));
        const float xv = to_f<TI>(*reinterpret_cast<const TI*>(tx + r * C::CPB * es));
        const float gv = to_f<TI>(*reinterpret_cast<const TI*>(tg + r * C::CPB * es));
        const float v = d * xv * st.advance(A2 * d);
        const float2 v2 = make_float2(v, v);
        const float4* B4 = reinterpret_cast<const float4*>(tbc + r * 2 * N);
        const float4* C4 = reinterpret_cast<const float4*>(tbc + r * 2 * N + N);
        float2 ya = make_float2(0.f, 0.f), yb = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < NS / 4; ++j) {
          const float4 bb = B4[j], cv = C4[j];
          st.g[2 * j] = __ffma2_rn(v2, make_float2(bb.x, bb.y), st.g[2 * j]);
          st.g[2 * j + 1] = __ffma2_rn(v2, make_float2(bb.z, bb.w), st.g[2 * j + 1]);
          ya = __ffma2_rn(make_float2(cv.x, cv.y), st.g[2 * j], ya);
          yb = __ffma2_rn(make_float2(cv.z, cv.w), st.g[2 * j + 1], yb);
        }
        float y = (ya.x + ya.y) + (yb.x + yb.y);
#pragma unroll
        for (int off = 1; off < TPC; off <<= 1) y += __shfl_xor_sync(0xffffffffu, y, off);
        if (slice == 0) yt[r * C::CPW + chw] = from_f<TI>(gv * ex2_approx(st.cl) * y);
      }
    }
    // release the input tile, then store this warp's y tile
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
    fence_proxy_async_smem();
    __syncwarp();
    const int ycol = blockIdx.x * C::CPB + warp * C::CPW;
    if (lane == 0 && ycol < p.Di) {  // a warp whose channels all lie past Di stores nothing
      tma_store_3d(&tmY, yt, ycol, k * C::ROWS, b);
      bulk_commit();
    }
  }
  if (lane == 0) bulk_wait_all();
  if (!ok && producer) {  // let the copies this warp has not consumed land before the CTA exits
    int never = 0;
    for (int t = k; t < static_cast<int>(issued); ++t)
      mbar_wait(&full[t % C::STAGES], (t / C::STAGES) & 1u, nullptr, &never, 100000000ull);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn scan_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 2-D map over [rows, cols] (row stride ld elements), box = bc x br, no swizzle.
bool map2d(CUtensorMap* m, const void* base, bool f32, long long rows, long long cols, long long ld, int bc, int br) {
  EncodeTiledFn fn = scan_encode_fn();
  if (!fn) return false;
  const int es = f32 ? 4 : 2;
  cuuint64_t gd[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t gs[1] = {static_cast<cuuint64_t>(ld) * es};
  cuuint32_t bx[2] = {static_cast<cuuint32_t>(bc), static_cast<cuuint32_t>(br)}, el[2] = {1, 1};
  return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
            gd, gs, bx, el, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over [batch][T][cols] (row stride ld elements), box = bc x br x 1, no swizzle.
bool map3d(CUtensorMap* m, const void* base, bool f32, int batch, int T, long long cols, long long ld, int bc,
           int br) {
  EncodeTiledFn fn = scan_encode_fn();
  if (!fn) return false;
  const int es = f32 ? 4 : 2;
  cuuint64_t gd[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(batch)};
  cuuint64_t gs[2] = {static_cast<cuuint64_t>(ld) * es, static_cast<cuuint64_t>(ld) * es * T};
  cuuint32_t bx[3] = {static_cast<cuuint32_t>(bc), static_cast<cuuint32_t>(br), 1}, el[3] = {1, 1, 1};
  return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
            gd, gs, bx, el, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename TI, int NS, int TPC>
cudaError_t launch_v5(const ScanDesc& s, cudaStream_t st) {
  using C = V5Cfg<TI, NS, TPC>;
  const bool f32 = sizeof(TI) == 4;
  CUtensorMap tx, td, tg, tb, ty;
  if (!map3d(&tx, s.x, f32, s.batch, s.T, s.d_inner, s.d_inner, C::CPB, C::ROWS) ||
      !map3d(&td, s.dt, f32, s.batch, s.T, s.d_inner, s.d_inner, C::CPB, C::ROWS) ||
      !map3d(&tg, s.gate, f32, s.batch, s.T, s.d_inner, s.d_inner, C::CPB, C::ROWS) ||
      !map3d(&tb, s.bc, true, s.batch, s.T, 2 * C::N, 2 * C::N, 2 * C::N, C::ROWS) ||
      !map3d(&ty, s.y, f32, s.batch, s.T, s.d_inner, s.y_ld, C::CPW, C::ROWS))
    return cudaErrorInvalidValue;
  static int attr_mask = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 31 && !(attr_mask & (1 << dev))) {
    cudaError_t e = cudaFuncSetAttribute(scan_v5_kernel<TI, NS, TPC>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_mask |= 1 << dev;
  }
  ScanParams p{s.x, s.dt, s.bc, s.gate, s.a_log, s.y, s.y_ld, s.T, s.d_inner, s.d_state};
  dim3 grid((s.d_inner + C::CPB - 1) / C::CPB, s.batch);
  scan_v5_kernel<TI, NS, TPC><<<grid, 32 * C::NWARP, C::SMEM, st>>>(tx, td, tg, tb, ty, p, s.status);
  return cudaGetLastError();
}

template <typename TI, int NS, int TPC, int NWT>
cudaError_t launch_one(const ScanDesc& s, cudaStream_t st) {
  constexpr int CPW = 32 / TPC;
  ScanParams p{s.x, s.dt, s.bc, s.gate, s.a_log, s.y, s.y_ld, s.T, s.d_inner, s.d_state};
  dim3 grid((s.d_inner + CPW - 1) / CPW, s.batch);
  scan_kernel<TI, NS, TPC, NWT><<<grid, 32 * NWT, 0, st>>>(p);
  return cudaGetLastError();
}

template <typename TI>
cudaError_t launch_t(const ScanDesc& s, cudaStream_t st) {
  // The TMA-staged single-pass kernel needs 16-byte aligned bases and row strides for
  // x, dt, gate, B|C and y; otherwise the per-channel kernel runs.
  auto a16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  const long long es = static_cast<long long>(sizeof(TI));
  const bool v5_ok = (s.d_inner * es) % 16 == 0 && (s.y_ld * es) % 16 == 0 && a16(s.x) && a16(s.dt) &&
                     a16(s.gate) && a16(s.bc) && a16(s.y);
  if (v5_ok) {
    switch (s.d_state) {
      case 16: return launch_v5<TI, 8, 2>(s, st);
      case 32: return launch_v5<TI, 16, 2>(s, st);
      case 64: return launch_v5<TI, 16, 4>(s, st);
      case 128: return launch_v5<TI, 32, 4>(s, st);
      default: break;  // N = 256: a B|C row exceeds one TMA box; per-channel kernel below
    }
  }
  switch (s.d_state) {
    case 16: return launch_one<TI, 16, 1, 16>(s, st);
    case 32: return launch_one<TI, 32, 1, 8>(s, st);
    case 64: return launch_one<TI, 32, 2, 8>(s, st);
    case 128: return launch_one<TI, 32, 4, 8>(s, st);
    case 256: return launch_one<TI, 32, 8, 8>(s, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_scan(const ScanDesc& s, cudaStream_t st) {
  if (s.batch <= 0 || s.T <= 0 || s.d_inner <= 0) return cudaSuccess;
  return s.bf16 ? launch_t<__nv_bfloat16>(s, st) : launch_t<float>(s, st);
}

}  // namespace hy
