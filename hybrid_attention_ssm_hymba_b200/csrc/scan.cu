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
