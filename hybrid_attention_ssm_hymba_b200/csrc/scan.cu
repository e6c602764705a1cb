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
// N <= 32: TMA-staged, scaled-state variant.
//
// Each lane owns two adjacent channels with all N state components (packed fp32x2
// pairs); a warp owns 64 channels (one 128-byte row segment per time step for bf16).
// A CTA walks T in segments of NWT * SUB steps; inside a segment warp w owns SUB
// consecutive steps and streams them through a private STAGES-deep ring of ROWS-step
// TMA tiles (x, dt, gate, B|C), so the recurrence never waits on a global load and
// the second pass re-reads data that is still in L2.
//
// Scaled state: with P_t = prod_{s<=t} exp(A dt_s) (since the last rescale) and
// g_t = h_t / P_t, the recurrence becomes g_t = g_{t-1} + (dt_t x_t / P_t) B_t and
// y_t = P_t (C_t . g_t): one FMA per state component per step instead of two.
// P is kept as its log2 (cl); when it would fall below 2^-60 the scale is folded
// back into g (g <- P g, cl <- 0), and a single step that decays by more than 2^-60
// simply restarts the state (its contribution from h_{t-1} is below 2^-60).
template <typename TI, int N>
struct PairCfg {
  static constexpr int NWT = 8;    // warps per CTA
  static constexpr int SUB = 64;   // steps per warp per segment
  static constexpr int SEG = NWT * SUB;
  static constexpr int ROWS = 8;   // time steps per staged tile
  static constexpr int STAGES = 3;
  static constexpr int CPW = 64;   // channels per warp (2 per lane)
  static constexpr int XB = ROWS * CPW * (int)sizeof(TI);  // bytes of one x / dt / gate tile
  static constexpr int BCB = ROWS * 2 * N * 4;              // bytes of one B|C tile
  static constexpr int STAGE_B = 3 * XB + BCB;
  static constexpr int WARP_B = STAGES * STAGE_B;
  static constexpr int RING_B = NWT * WARP_B;
  static constexpr int COMBINE_B = NWT * CPW * N * 4 + NWT * CPW * 4;
  static constexpr int AREA_B = RING_B > COMBINE_B ? RING_B : COMBINE_B;
  static constexpr int CARRY_B = 2 * CPW * N * 4;
  static constexpr int SMEM = AREA_B + CARRY_B + NWT * STAGES * 8 + 16 + 128;
};

template <typename TI> struct Pair2;
template <> struct Pair2<__nv_bfloat16> {
  static HY_DEV float2 ld(const uint8_t* p) {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    return make_float2(bf16lo(u), bf16hi(u));
  }
  static HY_DEV void st(__nv_bfloat16* p, float a, float b) { *reinterpret_cast<uint32_t*>(p) = pack_bf16(a, b); }
};
template <> struct Pair2<float> {
  static HY_DEV float2 ld(const uint8_t* p) { return *reinterpret_cast<const float2*>(p); }
  static HY_DEV void st(float* p, float a, float b) { *reinterpret_cast<float2*>(p) = make_float2(a, b); }
};

HY_DEV float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int NP>
struct ScaledState {
  float2 g[NP];
  float cl;  // log2 of the scale P
  HY_DEV void zero() {
#pragma unroll
    for (int i = 0; i < NP; ++i) g[i] = make_float2(0.f, 0.f);
    cl = 0.f;
  }
  // advance the scale by one step of log2-decay l2a; returns 1 / P_t
  HY_DEV float advance(float l2a) {
    float c = cl + l2a;
    if (c < -60.f) {  // rare: fold the scale into g
      const float P = ex2_approx(cl);
      const float2 P2 = make_float2(P, P);
#pragma unroll
      for (int i = 0; i < NP; ++i) g[i] = __fmul2_rn(g[i], P2);
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

// Fast path of one full ROWS-step tile.  First folds the running scale into g for
// every lane (g <- P g, P <- 1), then checks (warp-uniformly) that no lane's decay
// over the tile passes 2^-60, so that the scales of all its steps can be formed
// independently; returns false (slow, per-step guarded path) for a partial tile or
// an extreme decay.
template <typename TI, int N>
HY_DEV bool fast_tile(const uint8_t* tile, int lane, int rows, const float (&A2)[2], ScaledState<N / 2> (&st)[2]) {
  using C = PairCfg<TI, N>;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const float P = ex2_approx(st[q].cl);
    const float2 P2 = make_float2(P, P);
#pragma unroll
    for (int i = 0; i < N / 2; ++i) st[q].g[i] = __fmul2_rn(st[q].g[i], P2);
    st[q].cl = 0.f;
  }
  bool ok = rows == C::ROWS;
  if (ok) {
    float c[2] = {0.f, 0.f};
#pragma unroll
    for (int r = 0; r < C::ROWS; ++r) {
      const float2 dv = Pair2<TI>::ld(tile + C::XB + (r * C::CPW + 2 * lane) * sizeof(TI));
      c[0] = fmaf(A2[0], dv.x, c[0]);
      c[1] = fmaf(A2[1], dv.y, c[1]);
    }
    ok = c[0] >= -60.f && c[1] >= -60.f;
  }
  return __all_sync(0xffffffffu, ok);
}

// Four steps (rows h2 .. h2+3 of a staged tile) of the scaled-state recurrence with
// no fold needed: the four scales are formed up front (independent SFU ops), then the
// state chain runs; with EMIT the gated outputs y = gate P (C . g) are stored.
template <typename TI, int N, bool EMIT>
HY_DEV void step4(const uint8_t* tile, int lane, int h2, const float (&A2)[2], ScaledState<N / 2> (&st)[2],
                  float (&logdec)[2], TI* ybase, long long y_ld, int, bool w0, bool w1) {
  using C = PairCfg<TI, N>;
  float v[4][2], P[4][2], gate[4][2];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = h2 + k;
    const float2 xv = Pair2<TI>::ld(tile + (r * C::CPW + 2 * lane) * sizeof(TI));
    const float2 dv = Pair2<TI>::ld(tile + C::XB + (r * C::CPW + 2 * lane) * sizeof(TI));
    const float dq[2] = {dv.x, dv.y}, xq[2] = {xv.x, xv.y};
    if (EMIT) {
      const float2 gv = Pair2<TI>::ld(tile + 2 * C::XB + (r * C::CPW + 2 * lane) * sizeof(TI));
      gate[k][0] = gv.x;
      gate[k][1] = gv.y;
    }
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const float l2a = A2[q] * dq[q];
      if (!EMIT) logdec[q] += l2a;
      st[q].cl += l2a;
      v[k][q] = dq[q] * xq[q] * ex2_approx(-st[q].cl);
      if (EMIT) P[k][q] = ex2_approx(st[q].cl);
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = h2 + k;
    const float4* B4 = reinterpret_cast<const float4*>(tile + 3 * C::XB + r * 2 * N * 4);
    float2 q2[2], y2[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      q2[q] = make_float2(v[k][q], v[k][q]);
      y2[q] = make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < N / 4; ++j) {
      const float4 bb = B4[j];
      const float2 b01 = make_float2(bb.x, bb.y), b23 = make_float2(bb.z, bb.w);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        st[q].g[2 * j] = __ffma2_rn(q2[q], b01, st[q].g[2 * j]);
        st[q].g[2 * j + 1] = __ffma2_rn(q2[q], b23, st[q].g[2 * j + 1]);
      }
      if (EMIT) {
        const float4 cv = B4[N / 4 + j];
        const float2 c01 = make_float2(cv.x, cv.y), c23 = make_float2(cv.z, cv.w);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          y2[q] = __ffma2_rn(c01, st[q].g[2 * j], y2[q]);
          y2[q] = __ffma2_rn(c23, st[q].g[2 * j + 1], y2[q]);
        }
      }
    }
    if (EMIT) {
      TI* yrow = ybase + r * y_ld;
      const float ya = gate[k][0] * P[k][0] * (y2[0].x + y2[0].y);
      const float yb = gate[k][1] * P[k][1] * (y2[1].x + y2[1].y);
      if (w0 && w1) Pair2<TI>::st(yrow, ya, yb);
      else if (w0) yrow[0] = from_f<TI>(ya);
    }
  }
}

template <typename TI, int N>
__global__ void __launch_bounds__(256) scan_pair_kernel(const __grid_constant__ CUtensorMap tmX,
                                                        const __grid_constant__ CUtensorMap tmDT,
                                                        const __grid_constant__ CUtensorMap tmG,
                                                        const __grid_constant__ CUtensorMap tmBC,
                                                        const ScanParams p, unsigned* status) {
  using C = PairCfg<TI, N>;
  constexpr int NP = N / 2;
  extern __shared__ __align__(128) uint8_t smem[];
  float* s_carry = reinterpret_cast<float*>(smem + C::AREA_B);  // [2][CPW][N]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::AREA_B + C::CARRY_B);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + C::NWT * C::STAGES);
  float* s_hend = reinterpret_cast<float*>(smem);       // [NWT][CPW][N]  (aliases the ring)
  float* s_logdec = s_hend + C::NWT * C::CPW * N;       // [NWT][CPW]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int c0 = blockIdx.x * C::CPW + 2 * lane;  // this lane's first channel
  uint8_t* ring = smem + warp * C::WARP_B;
  uint64_t* my_full = full + warp * C::STAGES;

  if (threadIdx.x == 0) *abort_flag = 0;
  if (lane == 0)
    for (int s = 0; s < C::STAGES; ++s) mbar_init(&my_full[s], 1);
  for (int i = threadIdx.x; i < C::CPW * N; i += blockDim.x) s_carry[i] = 0.f;  // h = 0 before the first row
  fence_mbar_init();
  __syncthreads();

  float A2[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) A2[q] = c0 + q < p.Di ? -expf(p.a_log[c0 + q]) * 1.4426950408889634f : 0.f;
  const bool w0 = c0 < p.Di, w1 = c0 + 1 < p.Di;
  TI* Y = static_cast<TI*>(p.y);

  // Ring bookkeeping across segments and passes: the i-th tile issued by this warp
  // goes to slot i % STAGES and completes phase (i / STAGES) & 1 of that slot's
  // mbarrier; tiles are consumed in issue order.
  uint32_t issued = 0, consumed = 0;
  auto issue = [&](int grow, bool with_gate) {
    if (lane == 0) {
      const int slot = issued % C::STAGES;
      uint8_t* st = ring + slot * C::STAGE_B;
      uint64_t* bar = &my_full[slot];
      mbar_arrive_expect_tx(bar, (with_gate ? 3 : 2) * C::XB + C::BCB);
      const int col = blockIdx.x * C::CPW;
      tma_load_2d(st, &tmX, bar, col, grow);
      tma_load_2d(st + C::XB, &tmDT, bar, col, grow);
      if (with_gate) tma_load_2d(st + 2 * C::XB, &tmG, bar, col, grow);
      tma_load_2d(st + 3 * C::XB, &tmBC, bar, 0, grow);
    }
    ++issued;
  };
  auto wait_tile = [&]() -> bool {
    return __all_sync(0xffffffffu,
                      mbar_wait(&my_full[consumed % C::STAGES], (consumed / C::STAGES) & 1u, status, abort_flag));
  };
  auto drain = [&]() {  // after an abort: let this warp's copies in flight land
    int never = 0;
    if (lane == 0)
      for (uint32_t i = consumed; i < issued; ++i)
        mbar_wait(&my_full[i % C::STAGES], (i / C::STAGES) & 1u, nullptr, &never, 100000000ull);
    __syncwarp();
  };

  bool ok = true;
  ScaledState<NP> st[2];
  int seg_id = 0;
  for (int seg0 = 0; seg0 < p.T; seg0 += C::SEG, ++seg_id) {
    const int t0 = min(p.T, seg0 + warp * C::SUB), t1 = min(p.T, min(seg0 + C::SEG, t0 + C::SUB));
    const int n_tiles = (t1 - t0 + C::ROWS - 1) / C::ROWS;
    const int grow0 = b * p.T + t0;
    // ---------------- pass 1: local scan from h = 0 -> end state and total log2-decay
    float logdec[2] = {0.f, 0.f};
#pragma unroll
    for (int q = 0; q < 2; ++q) st[q].zero();
    for (int k = 0; ok && k < C::STAGES - 1 && k < n_tiles; ++k) issue(grow0 + k * C::ROWS, false);
    for (int k = 0; ok && k < n_tiles; ++k) {
      __syncwarp();
      if (k + C::STAGES - 1 < n_tiles) issue(grow0 + (k + C::STAGES - 1) * C::ROWS, false);
      const uint8_t* tile = ring + (consumed % C::STAGES) * C::STAGE_B;
      if (!wait_tile()) {
        ok = false;
        break;
      }
      ++consumed;
      const int rows = min(C::ROWS, t1 - t0 - k * C::ROWS);
      if (fast_tile<TI, N>(tile, lane, rows, A2, st)) {
#pragma unroll
        for (int h2 = 0; h2 < C::ROWS; h2 += 4) step4<TI, N, false>(tile, lane, h2, A2, st, logdec, nullptr, 0, 0, false, false);
      } else {
        for (int r = 0; r < rows; ++r) {
          const float2 xv = Pair2<TI>::ld(tile + (r * C::CPW + 2 * lane) * sizeof(TI));
          const float2 dv = Pair2<TI>::ld(tile + C::XB + (r * C::CPW + 2 * lane) * sizeof(TI));
          const float4* B4 = reinterpret_cast<const float4*>(tile + 3 * C::XB + r * 2 * N * 4);
          const float dq[2] = {dv.x, dv.y}, xq[2] = {xv.x, xv.y};
          float2 q2[2];
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const float l2a = A2[q] * dq[q];
            logdec[q] += l2a;
            const float v = dq[q] * xq[q] * st[q].advance(l2a);
            q2[q] = make_float2(v, v);
          }
#pragma unroll
          for (int j = 0; j < N / 4; ++j) {
            const float4 bb = B4[j];
            const float2 b01 = make_float2(bb.x, bb.y), b23 = make_float2(bb.z, bb.w);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              st[q].g[2 * j] = __ffma2_rn(q2[q], b01, st[q].g[2 * j]);
              st[q].g[2 * j + 1] = __ffma2_rn(q2[q], b23, st[q].g[2 * j + 1]);
            }
          }
        }
      }
    }
    if (!ok) drain();
    __syncthreads();  // the ring area becomes the combine area
    // local end state h_end = P g
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const float P = ex2_approx(st[q].cl);
      const float2 P2 = make_float2(P, P);
      float2* dst = reinterpret_cast<float2*>(s_hend + (warp * C::CPW + 2 * lane + q) * N);
#pragma unroll
      for (int i = 0; i < NP; ++i) dst[i] = __fmul2_rn(st[q].g[i], P2);
      s_logdec[warp * C::CPW + 2 * lane + q] = logdec[q];
    }
    __syncthreads();
    // ---------------- combine: state entering this warp's steps (chained from the
    // segment's carry-in), and the last warp also forms the next segment's carry-in
    const float* carry_in = s_carry + (seg_id & 1) * C::CPW * N;
    float* carry_out = s_carry + ((seg_id + 1) & 1) * C::CPW * N;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int ch = 2 * lane + q;
      const float2* cin = reinterpret_cast<const float2*>(carry_in + ch * N);
#pragma unroll
      for (int i = 0; i < NP; ++i) st[q].g[i] = cin[i];
      st[q].cl = 0.f;
      const int kmax = (warp == C::NWT - 1) ? C::NWT : warp;
      for (int k = 0; k < kmax; ++k) {
        if (k == warp) {  // last warp: its own entry state is complete; store it, then go on
          float2* tmp = reinterpret_cast<float2*>(carry_out + ch * N);
#pragma unroll
          for (int i = 0; i < NP; ++i) tmp[i] = st[q].g[i];
        }
        const float dec = ex2_approx(s_logdec[k * C::CPW + ch]);
        const float2 dec2 = make_float2(dec, dec);
        const float2* hk = reinterpret_cast<const float2*>(s_hend + (k * C::CPW + ch) * N);
#pragma unroll
        for (int i = 0; i < NP; ++i) st[q].g[i] = __ffma2_rn(dec2, st[q].g[i], hk[i]);
      }
      if (warp == C::NWT - 1) {  // g = carry-out (end of segment); restore own entry state
        float2* co = reinterpret_cast<float2*>(carry_out + ch * N);
#pragma unroll
        for (int i = 0; i < NP; ++i) {
          const float2 own = co[i];
          co[i] = st[q].g[i];
          st[q].g[i] = own;
        }
      }
    }
    fence_proxy_async_smem();  // generic accesses to the ring area before the copies below
    __syncthreads();
    // ---------------- pass 2: rescan from the carried state, emit y = gate (C . h)
    for (int k = 0; ok && k < C::STAGES - 1 && k < n_tiles; ++k) issue(grow0 + k * C::ROWS, true);
    for (int k = 0; ok && k < n_tiles; ++k) {
      __syncwarp();
      if (k + C::STAGES - 1 < n_tiles) issue(grow0 + (k + C::STAGES - 1) * C::ROWS, true);
      const uint8_t* tile = ring + (consumed % C::STAGES) * C::STAGE_B;
      if (!wait_tile()) {
        ok = false;
        break;
      }
      ++consumed;
      const int rows = min(C::ROWS, t1 - t0 - k * C::ROWS);
      if (fast_tile<TI, N>(tile, lane, rows, A2, st)) {
        float ld_unused[2] = {0.f, 0.f};
        TI* ybase = Y + (static_cast<long long>(grow0) + k * C::ROWS) * p.y_ld + c0;
#pragma unroll
        for (int h2 = 0; h2 < C::ROWS; h2 += 4)
          step4<TI, N, true>(tile, lane, h2, A2, st, ld_unused, ybase, p.y_ld, 0, w0, w1);
        continue;
      }
      for (int r = 0; r < rows; ++r) {
        const float2 xv = Pair2<TI>::ld(tile + (r * C::CPW + 2 * lane) * sizeof(TI));
        const float2 dv = Pair2<TI>::ld(tile + C::XB + (r * C::CPW + 2 * lane) * sizeof(TI));
        const float2 gv = Pair2<TI>::ld(tile + 2 * C::XB + (r * C::CPW + 2 * lane) * sizeof(TI));
        const float4* B4 = reinterpret_cast<const float4*>(tile + 3 * C::XB + r * 2 * N * 4);
        const float4* C4 = B4 + N / 4;
        const float dq[2] = {dv.x, dv.y}, xq[2] = {xv.x, xv.y};
        float2 q2[2], y2[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const float v = dq[q] * xq[q] * st[q].advance(A2[q] * dq[q]);
          q2[q] = make_float2(v, v);
          y2[q] = make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int j = 0; j < N / 4; ++j) {
          const float4 bb = B4[j], cv = C4[j];
          const float2 b01 = make_float2(bb.x, bb.y), b23 = make_float2(bb.z, bb.w);
          const float2 c01 = make_float2(cv.x, cv.y), c23 = make_float2(cv.z, cv.w);
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            st[q].g[2 * j] = __ffma2_rn(q2[q], b01, st[q].g[2 * j]);
            st[q].g[2 * j + 1] = __ffma2_rn(q2[q], b23, st[q].g[2 * j + 1]);
            y2[q] = __ffma2_rn(c01, st[q].g[2 * j], y2[q]);
            y2[q] = __ffma2_rn(c23, st[q].g[2 * j + 1], y2[q]);
          }
        }
        const long long row = static_cast<long long>(grow0) + k * C::ROWS + r;
        TI* yrow = Y + row * p.y_ld + c0;
        const float ya = gv.x * ex2_approx(st[0].cl) * (y2[0].x + y2[0].y);
        const float yb = gv.y * ex2_approx(st[1].cl) * (y2[1].x + y2[1].y);
        if (w0 && w1) Pair2<TI>::st(yrow, ya, yb);
        else if (w0) yrow[0] = from_f<TI>(ya);
      }
    }
    if (!ok) drain();
    __syncthreads();  // carry-out visible; the ring area is reused by the next segment's pass 1
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

template <typename TI, int N>
cudaError_t launch_pair(const ScanDesc& s, cudaStream_t st) {
  using C = PairCfg<TI, N>;
  const bool f32 = sizeof(TI) == 4;
  const long long rows = static_cast<long long>(s.batch) * s.T;
  CUtensorMap tx, td, tg, tb;
  if (!map2d(&tx, s.x, f32, rows, s.d_inner, s.d_inner, C::CPW, C::ROWS) ||
      !map2d(&td, s.dt, f32, rows, s.d_inner, s.d_inner, C::CPW, C::ROWS) ||
      !map2d(&tg, s.gate, f32, rows, s.d_inner, s.d_inner, C::CPW, C::ROWS) ||
      !map2d(&tb, s.bc, true, rows, 2 * N, 2 * N, 2 * N, C::ROWS))
    return cudaErrorInvalidValue;
  static int attr_mask = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 31 && !(attr_mask & (1 << dev))) {
    cudaError_t e = cudaFuncSetAttribute(scan_pair_kernel<TI, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_mask |= 1 << dev;
  }
  ScanParams p{s.x, s.dt, s.bc, s.gate, s.a_log, s.y, s.y_ld, s.T, s.d_inner, s.d_state};
  dim3 grid((s.d_inner + C::CPW - 1) / C::CPW, s.batch);
  scan_pair_kernel<TI, N><<<grid, 32 * C::NWT, C::SMEM, st>>>(tx, td, tg, tb, p, s.status);
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
  // The TMA-staged pair kernel needs 16-byte aligned bases and row strides for x, dt,
  // gate, B|C, and 2-channel aligned output stores; otherwise the per-channel kernel runs.
  auto a16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  const bool pair_ok = (s.d_inner * static_cast<int>(sizeof(TI))) % 16 == 0 && a16(s.x) && a16(s.dt) &&
                       a16(s.gate) && a16(s.bc) && (s.y_ld % 2) == 0 &&
                       (reinterpret_cast<uintptr_t>(s.y) % (2 * sizeof(TI))) == 0;
  switch (s.d_state) {
    case 16: return pair_ok ? launch_pair<TI, 16>(s, st) : launch_one<TI, 16, 1, 16>(s, st);
    case 32: return pair_ok ? launch_pair<TI, 32>(s, st) : launch_one<TI, 32, 1, 8>(s, st);
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
