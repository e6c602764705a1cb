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

// Launch shapes of the main kernel (lanes per channel, channels per lane) for the two
// state sizes of the workloads.
#ifndef HY_SCAN16_TPC
#define HY_SCAN16_TPC 1
#define HY_SCAN16_CPL 2
#endif
// bf16 with d_state = 16 runs the tensor-core block form (scan_tc.cu) by default.
#ifndef HY_SCAN_TC
#define HY_SCAN_TC 1
#endif
#ifndef HY_SCAN128_TPC
#define HY_SCAN128_TPC 4
#define HY_SCAN128_CPL 2
#endif

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
  float* h_out;  // [batch, Di, N] state after the last row, or nullptr
  int t0;                 // first row scanned
  const float* h0;        // [Di, N] state entering row t0 (sequence b at h0 + b * h0_bstride), or nullptr
  long long h0_bstride;
};

// The state entering row t0 for NS components [n0, n0 + NS) of channel c of sequence b.
HY_DEV void load_h0(const ScanParams& p, int b, int c, int n0, int NS, float* h) {
  for (int n = 0; n < NS; ++n) h[n] = p.h0 ? p.h0[b * p.h0_bstride + static_cast<long long>(c) * p.N + n0 + n] : 0.f;
}

template <typename TI, int NS, int TPC, int NWT>
__global__ void __launch_bounds__(32 * NWT) scan_kernel(const ScanParams p) {
  pdl_trigger();
  pdl_wait();
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
  const int Lc = (p.T - p.t0 + NWT - 1) / NWT;
  const int t0 = min(p.T, p.t0 + warp * Lc), t1 = min(p.T, t0 + Lc);
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

  // ---------------- combine: state entering this warp's chunk (from the state entering row t0)
  {
    float hz[NS];
    load_h0(p, b, cc, n0, NS, hz);
#pragma unroll
    for (int i = 0; i < NP; ++i) h[i] = make_float2(hz[2 * i], hz[2 * i + 1]);
  }
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
  // the last chunk's warp ends at row T - 1 (an empty chunk keeps its entry state)
  if (p.h_out && valid && warp == NWT - 1) {
    float* ho = p.h_out + (static_cast<long long>(b) * p.Di + c) * N + n0;
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      ho[2 * i] = h[i].x;
      ho[2 * i + 1] = h[i].y;
    }
  }
}

// ---------------------------------------------------------------------------------
// Main scan kernel: warp-private pipelines, optional split of T into chunks.
//
// A lane owns CPL adjacent channels and NS = N / TPC of their state components (TPC
// lanes per channel); partial dot products are reduced over the TPC lanes with
// shuffles.  Every warp streams its own STAGES-deep ring of ROWS-step TMA tiles (x, dt,
// gate of its CPW channels and the full B|C rows), refilled by its own lane 0, and
// writes y through a double-buffered smem tile and TMA stores.  A CTA holds G channel
// groups x S time chunks of one sequence (G * S warps).  With S = 1 each warp scans all
// T steps of its channels once.  With S > 1 the warps of a group take consecutive
// chunks: pass 1 scans each chunk but the last from h = 0 for its end state only
// (state update, no output, no gate or C reads); the end states meet in shared
// memory, where chunk k forms its entry state c_k = D_{k-1} c_{k-1} + h_end_{k-1}
// (D = the chunk's total decay); pass 2 rescans every chunk from its entry state and
// emits y.  S is chosen per launch so that the SM sub-partitions have enough warps.
// Tensor maps are 3-D ([batch][T][cols]): no tile crosses a sequence end, rows past T
// load as zeros (dt = 0 leaves the state unchanged) and are clipped on store.
//
// Scaled state: with P_t = prod exp(A dt_s) since the last rescale and g = h / P,
// g_t = g_{t-1} + (dt_t x_t / P_t) B_t and y_t = P_t (C_t . g_t).  The output is
// formed as y_t = P_t (C_t . g_{t-1} + v_t (C_t . B_t)), v_t = dt_t x_t / P_t, so that it
// reads only the previous state and never waits on this step's update; the row dot
// product C_t . B_t is shared by all channels and computed once per tile row.
// -log2 P is kept per channel (ncl) and folded back into g every block of BLK steps;
// a block whose decay would take P below 2^-60 runs the per-step path that folds on
// demand and restarts the state after a single step decaying by more than 2^-60.
//
// B|C reads: lanes of different slices read different 16-byte chunks of the same row;
// slice s visits its chunks in an order rotated by (s * NS / 32), which puts the
// slices' chunks in distinct shared-memory banks.
template <typename TI, int N, int TPC, int CPL>
struct WCfg {
  static constexpr int NS = N / TPC;            // state components per lane and channel
  static constexpr int NP = NS / 2;             // packed fp32x2 pairs
  static constexpr int NQ = NS / 4;             // 16-byte chunks of B (and of C) per lane
  static constexpr int CPW = (32 / TPC) * CPL;  // channels per warp
  static constexpr int BLK = NQ * CPL <= 4 ? 16 : 8;  // steps per unrolled block (registers)
  static constexpr int ROWS = (N == 16 && sizeof(TI) == 2 && CPL == 1) ? 32 : (N <= 32 ? 16 : 8);
  static constexpr int STAGES = (N <= 32 && TPC == 1) ? (CPL == 1 ? 4 : 2) : 3;
  static constexpr int LPR = 32 / ROWS;               // lanes per row for C . B
  static constexpr int XB = ROWS * CPW * (int)sizeof(TI);  // one x / dt / gate tile
  static constexpr int BCB = ROWS * 2 * N * 4;              // one B|C tile
  static constexpr int STAGE_B = 3 * XB + BCB;
  static constexpr int YB = ROWS * CPW * (int)sizeof(TI);   // one y tile
  static constexpr int WARP_B = (STAGES * STAGE_B + 2 * YB + STAGES * 8 + 16 + 127) / 128 * 128;
  static constexpr int MAX_WARPS = 8;
  static constexpr int HEND_B = 32 * CPL * (NS + 1) * 4;    // a warp's end state + log-decay
  static_assert(ROWS % BLK == 0 && 32 % ROWS == 0, "tile rows");
  static_assert(HEND_B <= STAGE_B, "the end state is published in ring slot 0");
  static_assert(4 * WARP_B + 128 <= 227 * 1024, "shared memory per CTA");
};

// CPL adjacent channels of one row: load from a shared address, store to a pointer.
template <typename TI, int CPL> struct ChanLd;
template <> struct ChanLd<__nv_bfloat16, 1> {
  static HY_DEV void ld(uint32_t a, float (&v)[1]) { v[0] = __uint_as_float(lds_u16(a) << 16); }
  static HY_DEV void st(uint8_t* p, const float (&v)[1]) { *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(v[0]); }
};
template <> struct ChanLd<__nv_bfloat16, 2> {
  static HY_DEV void ld(uint32_t a, float (&v)[2]) {
    const uint32_t u = lds_u32(a);
    v[0] = bf16lo(u);
    v[1] = bf16hi(u);
  }
  static HY_DEV void st(uint8_t* p, const float (&v)[2]) { *reinterpret_cast<uint32_t*>(p) = pack_bf16(v[0], v[1]); }
};
template <> struct ChanLd<float, 1> {
  static HY_DEV void ld(uint32_t a, float (&v)[1]) { v[0] = lds_f32(a); }
  static HY_DEV void st(uint8_t* p, const float (&v)[1]) { *reinterpret_cast<float*>(p) = v[0]; }
};
template <> struct ChanLd<float, 2> {
  static HY_DEV void ld(uint32_t a, float (&v)[2]) {
    const float2 f = lds_f2(a);
    v[0] = f.x;
    v[1] = f.y;
  }
  static HY_DEV void st(uint8_t* p, const float (&v)[2]) { *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]); }
};

struct SplitParams {
  int S;       // time chunks per channel group (warps per group)
  int G;       // channel groups per CTA
  int ctiles;  // tiles per chunk
};

template <typename TI, int N, int TPC, int CPL>
__global__ void __launch_bounds__(256) scan_w_kernel(const __grid_constant__ CUtensorMap tmX,
                                                     const __grid_constant__ CUtensorMap tmDT,
                                                     const __grid_constant__ CUtensorMap tmG,
                                                     const __grid_constant__ CUtensorMap tmBC,
                                                     const __grid_constant__ CUtensorMap tmY, const ScanParams p,
                                                     const SplitParams sp, unsigned* status) {
  using C = WCfg<TI, N, TPC, CPL>;
  constexpr int NS = C::NS, NP = C::NP, NQ = C::NQ, CPW = C::CPW;
  constexpr uint32_t es = sizeof(TI);
  extern __shared__ __align__(128) uint8_t smem_raw[];
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int grp = warp / sp.S, chunk = warp % sp.S;
  const int wcol = (blockIdx.x * sp.G + grp) * CPW;  // first channel of this warp
  const bool active = wcol < p.Di;                   // inactive warps still meet the CTA barriers
  const int n_tiles = (p.T - p.t0 + C::ROWS - 1) / C::ROWS;   // tiles of rows [t0, T)
  const int k_begin = min(n_tiles, chunk * sp.ctiles), k_end = min(n_tiles, k_begin + sp.ctiles);

  uint8_t* wsm = smem_raw + warp * C::WARP_B;
  const uint32_t ring = smem_u32(wsm);
  uint8_t* ybuf = wsm + C::STAGES * C::STAGE_B;  // [2][ROWS][CPW]
  uint64_t* full = reinterpret_cast<uint64_t*>(ybuf + 2 * C::YB);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + C::STAGES);

  if (lane == 0) {
    for (int s = 0; s < C::STAGES; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  // Ring bookkeeping across both passes: the i-th tile this warp issues goes to slot
  // i % STAGES and completes phase (i / STAGES) & 1 there; tiles are consumed in order.
  uint32_t issued = 0, consumed = 0;  // (issued is meaningful on lane 0)
  auto issue = [&](int k, bool with_gate) {  // lane 0: time tile k
    const int slot = issued % C::STAGES;
    uint8_t* st = wsm + slot * C::STAGE_B;
    mbar_arrive_expect_tx(&full[slot], (with_gate ? 3 : 2) * C::XB + C::BCB);
    const int t = p.t0 + k * C::ROWS;
    tma_load_3d(st, &tmX, &full[slot], wcol, t, b);
    tma_load_3d(st + C::XB, &tmDT, &full[slot], wcol, t, b);
    if (with_gate) tma_load_3d(st + 2 * C::XB, &tmG, &full[slot], wcol, t, b);
    tma_load_3d(st + 3 * C::XB, &tmBC, &full[slot], 0, t, b);
    ++issued;
  };
  bool ok = true;
  auto wait_tile = [&]() -> bool {
    const bool r = __all_sync(0xffffffffu, mbar_wait(&full[consumed % C::STAGES], (consumed / C::STAGES) & 1u,
                                                     status, abort_flag));
    ++consumed;
    return r;
  };

  const int cg = lane / TPC, slice = lane % TPC;
  const int ccol = cg * CPL;  // first channel of this lane within the warp
  const int c0 = wcol + ccol;
  const int n0 = slice * NS;
  const int rot = (slice * NS / 32) & (NQ - 1);
  float A2[CPL];  // A in log2 units: exp(A dt) = exp2(A2 dt)
#pragma unroll
  for (int q = 0; q < CPL; ++q) A2[q] = (active && c0 + q < p.Di) ? -expf(p.a_log[c0 + q]) * 1.4426950408889634f : 0.f;

  float2 g[CPL][NP];
  float ncl[CPL];  // -log2 of the running scale P
#pragma unroll
  for (int q = 0; q < CPL; ++q) {
#pragma unroll
    for (int i = 0; i < NP; ++i) g[q][i] = make_float2(0.f, 0.f);
    ncl[q] = 0.f;
  }
  const bool ywriter = slice == 0;
  // the state entering row t0: the entry state of a single chunk, or the start of the
  // chunk combine below
  // g[q][2j], g[q][2j + 1] hold state components n0 + ((j + rot) % NQ) * 4 + {0, 1}, {2, 3}
  // (the lane's 16-byte chunks are visited in a rotated order, see load_b)
  float2 g0[CPL][NP];
#pragma unroll
  for (int q = 0; q < CPL; ++q) {
    float hz[NS];
    load_h0(p, b, (active && c0 + q < p.Di) ? c0 + q : 0, n0, NS, hz);
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
      const int e = ((j + rot) & (NQ - 1)) * 4;
      g0[q][2 * j] = make_float2(hz[e], hz[e + 1]);
      g0[q][2 * j + 1] = make_float2(hz[e + 2], hz[e + 3]);
    }
  }
  if (sp.S == 1) {
#pragma unroll
    for (int q = 0; q < CPL; ++q)
#pragma unroll
      for (int i = 0; i < NP; ++i) g[q][i] = g0[q][i];
  }

  auto load_b = [&](uint32_t row_addr, float4 (&bq)[NQ]) {
#pragma unroll
    for (int j = 0; j < NQ; ++j) bq[j] = lds_f4(row_addr + (n0 + ((j + rot) & (NQ - 1)) * 4) * 4);
  };
  auto load_bc = [&](uint32_t row_addr, float4 (&bq)[NQ], float4 (&cq)[NQ]) {
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
      const uint32_t off = (n0 + ((j + rot) & (NQ - 1)) * 4) * 4;
      bq[j] = lds_f4(row_addr + off);
      cq[j] = lds_f4(row_addr + N * 4 + off);
    }
  };
  // g_t = g_{t-1} + v_t B_t
  auto update = [&](const float4 (&bq)[NQ], const float (&v)[CPL]) {
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
      const float2 b01 = make_float2(bq[j].x, bq[j].y), b23 = make_float2(bq[j].z, bq[j].w);
#pragma unroll
      for (int q = 0; q < CPL; ++q) {
        const float2 v2 = make_float2(v[q], v[q]);
        g[q][2 * j] = __ffma2_rn(v2, b01, g[q][2 * j]);
        g[q][2 * j + 1] = __ffma2_rn(v2, b23, g[q][2 * j + 1]);
      }
    }
  };
  // y = C_t . g_{t-1} + v_t (C_t . B_t) (the partial dot reduced over the slices), then
  // g_t = g_{t-1} + v_t B_t.  Both read only the previous state.
  auto step_core = [&](const float4 (&bq)[NQ], const float4 (&cq)[NQ], const float (&v)[CPL], float cb,
                       float (&y)[CPL]) {
    float2 ya[CPL], yb[CPL];
#pragma unroll
    for (int q = 0; q < CPL; ++q) {
      ya[q] = make_float2(0.f, 0.f);
      yb[q] = make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
      const float2 c01 = make_float2(cq[j].x, cq[j].y), c23 = make_float2(cq[j].z, cq[j].w);
#pragma unroll
      for (int q = 0; q < CPL; ++q) {
        ya[q] = __ffma2_rn(c01, g[q][2 * j], ya[q]);
        yb[q] = __ffma2_rn(c23, g[q][2 * j + 1], yb[q]);
      }
    }
    update(bq, v);
#pragma unroll
    for (int q = 0; q < CPL; ++q) {
      float sum = (ya[q].x + ya[q].y) + (yb[q].x + yb[q].y);
#pragma unroll
      for (int off = 1; off < TPC; off <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      y[q] = fmaf(v[q], cb, sum);
    }
  };
  // one step of the per-step (extreme decay) path: fold on demand, restart after a single
  // step decaying past 2^-60; returns v and keeps ncl
  auto slow_scalars = [&](const float (&dv)[CPL], const float (&xv)[CPL], float (&vv)[CPL], float (&lsum)[CPL]) {
#pragma unroll
    for (int q = 0; q < CPL; ++q) {
      const float l = -A2[q] * dv[q];  // >= 0
      lsum[q] += l;
      float c = ncl[q] + l;
      if (c > 60.f) {
        const float Pf = ex2_approx(-ncl[q]);
        const float2 P2 = make_float2(Pf, Pf);
#pragma unroll
        for (int i = 0; i < NP; ++i) g[q][i] = __fmul2_rn(g[q][i], P2);
        if (l > 60.f) {
#pragma unroll
          for (int i = 0; i < NP; ++i) g[q][i] = make_float2(0.f, 0.f);
          c = 0.f;
        } else {
          c = l;
        }
      }
      ncl[q] = c;
      vv[q] = dv[q] * xv[q] * ex2_approx(c);
    }
  };
  auto fold = [&]() {
#pragma unroll
    for (int q = 0; q < CPL; ++q) {
      const float P = ex2_approx(-ncl[q]);
      const float2 P2 = make_float2(P, P);
#pragma unroll
      for (int i = 0; i < NP; ++i) g[q][i] = __fmul2_rn(g[q][i], P2);
      ncl[q] = 0.f;
    }
  };
  // B|C rows are prefetched one step ahead when the registers allow it
  constexpr bool kPrefetch = NQ * CPL <= 4;

  // ======================== pass 1: end state of this chunk (every chunk but the last)
  float ltot[CPL];  // the chunk's total decay, -log2 D
#pragma unroll
  for (int q = 0; q < CPL; ++q) ltot[q] = 0.f;
  const bool pass1 = active && sp.S > 1 && chunk < sp.S - 1;
  if (pass1) {
    if (lane == 0)
      for (int k = k_begin; k < k_end && k < k_begin + C::STAGES; ++k) issue(k, false);
    for (int k = k_begin; k < k_end; ++k) {
      if (!wait_tile()) {
        ok = false;
        break;
      }
      const uint32_t tile = ring + ((consumed - 1) % C::STAGES) * C::STAGE_B;
      const uint32_t tx = tile + ccol * es, td = tile + C::XB + ccol * es, tbc = tile + 3 * C::XB;
#pragma unroll 1
      for (int r0 = 0; r0 < C::ROWS; r0 += C::BLK) {
        fold();
        float v[C::BLK][CPL];
        bool fast = true;
        {
          float nc[CPL];
#pragma unroll
          for (int q = 0; q < CPL; ++q) nc[q] = 0.f;
#pragma unroll
          for (int s = 0; s < C::BLK; ++s) {
            float dv[CPL], xv[CPL];
            const uint32_t ro = (r0 + s) * CPW * es;
            ChanLd<TI, CPL>::ld(td + ro, dv);
            ChanLd<TI, CPL>::ld(tx + ro, xv);
#pragma unroll
            for (int q = 0; q < CPL; ++q) {
              nc[q] = fmaf(-A2[q], dv[q], nc[q]);
              v[s][q] = dv[q] * xv[q] * ex2_approx(nc[q]);
            }
          }
#pragma unroll
          for (int q = 0; q < CPL; ++q) {
            fast = fast && nc[q] <= 60.f;
            ncl[q] = nc[q];
          }
        }
        if (__all_sync(0xffffffffu, fast)) {
#pragma unroll
          for (int q = 0; q < CPL; ++q) ltot[q] += ncl[q];
          float4 bq[2][NQ];
          load_b(tbc + r0 * 2 * N * 4, bq[0]);
#pragma unroll
          for (int s = 0; s < C::BLK; ++s) {
            if (s + 1 < C::BLK) load_b(tbc + (r0 + s + 1) * 2 * N * 4, bq[(s + 1) & 1]);
            update(bq[s & 1], v[s]);
          }
        } else {
#pragma unroll
          for (int q = 0; q < CPL; ++q) ncl[q] = 0.f;
#pragma unroll 1
          for (int s = 0; s < C::BLK; ++s) {
            float dv[CPL], xv[CPL], vv[CPL];
            const uint32_t ro = (r0 + s) * CPW * es;
            ChanLd<TI, CPL>::ld(td + ro, dv);
            ChanLd<TI, CPL>::ld(tx + ro, xv);
            slow_scalars(dv, xv, vv, ltot);
            float4 bq[NQ];
            load_b(tbc + (r0 + s) * 2 * N * 4, bq);
            update(bq, vv);
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && k + C::STAGES < k_end) issue(k + C::STAGES, false);
    }
  }
  // ======================== combine: entry state of every chunk
  if (sp.S > 1) {
    // the end state h = P g and -log2 D, published in ring slot 0 (no copy in flight now)
    float* pub = reinterpret_cast<float*>(wsm) + lane * CPL * (NS + 1);
    if (pass1) {
#pragma unroll
      for (int q = 0; q < CPL; ++q) {
        const float P = ex2_approx(-ncl[q]);
#pragma unroll
        for (int i = 0; i < NP; ++i) {
          pub[q * (NS + 1) + 2 * i] = g[q][i].x * P;
          pub[q * (NS + 1) + 2 * i + 1] = g[q][i].y * P;
        }
        pub[q * (NS + 1) + NS] = ltot[q];
      }
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < CPL; ++q) {
#pragma unroll
      for (int i = 0; i < NP; ++i) g[q][i] = g0[q][i];
      ncl[q] = 0.f;
    }
    for (int j = 0; j < chunk; ++j) {  // c_{j+1} = D_j c_j + h_end_j
      const float* src = reinterpret_cast<const float*>(smem_raw + (grp * sp.S + j) * C::WARP_B) +
                         lane * CPL * (NS + 1);
#pragma unroll
      for (int q = 0; q < CPL; ++q) {
        const float D = ex2_approx(-src[q * (NS + 1) + NS]);
        const float2 D2 = make_float2(D, D);
#pragma unroll
        for (int i = 0; i < NP; ++i)
          g[q][i] = __ffma2_rn(D2, g[q][i], make_float2(src[q * (NS + 1) + 2 * i], src[q * (NS + 1) + 2 * i + 1]));
      }
    }
    fence_proxy_async_smem();  // the published values are read before copies overwrite slot 0
    __syncthreads();
  }

  // ======================== pass 2: scan the chunk from its entry state, emit y
  if (active && ok) {
    if (lane == 0)
      for (int k = k_begin; k < k_end && k < k_begin + C::STAGES; ++k) issue(k, true);
    for (int k = k_begin; k < k_end; ++k) {
      if (!wait_tile()) {
        ok = false;
        break;
      }
      const int slot = (consumed - 1) % C::STAGES;
      const uint32_t tile = ring + slot * C::STAGE_B;
      const uint32_t tx = tile + ccol * es;
      const uint32_t td = tile + C::XB + ccol * es;
      const uint32_t tg = tile + 2 * C::XB + ccol * es;
      const uint32_t tbc = tile + 3 * C::XB;
      uint8_t* yt = ybuf + (k & 1) * C::YB;  // this warp's y tile [ROWS][CPW]
      if (lane == 0) bulk_wait_read1();      // the store of tile k-2 has read this buffer
      __syncwarp();

      // C_t . B_t of the tile's rows: LPR lanes per row, chunks rotated by row (banks)
      float cb_row;
      {
        constexpr int CPP = (N / 4) / C::LPR;  // 16-byte chunks per lane
        const int row = lane / C::LPR, part = lane % C::LPR;
        const uint32_t ra = tbc + row * 2 * N * 4;
        float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < CPP; ++j) {
          const uint32_t off = (part * CPP + ((j + row) & (CPP - 1))) * 16;
          const float4 bb = lds_f4(ra + off), cc = lds_f4(ra + N * 4 + off);
          a0 = __ffma2_rn(make_float2(bb.x, bb.y), make_float2(cc.x, cc.y), a0);
          a1 = __ffma2_rn(make_float2(bb.z, bb.w), make_float2(cc.z, cc.w), a1);
        }
        cb_row = (a0.x + a0.y) + (a1.x + a1.y);
#pragma unroll
        for (int off = 1; off < C::LPR; off <<= 1) cb_row += __shfl_xor_sync(0xffffffffu, cb_row, off);
      }

      // blocks of BLK steps: fold the scale into g, then either the unrolled fast block
      // (every scalar of the block's steps first -- loads, decay chain, SFU -- then the
      // state chain with B|C prefetched one step ahead) or, when some channel's decay
      // over the block passes 2^-60, the per-step path.
#pragma unroll 1
      for (int r0 = 0; r0 < C::ROWS; r0 += C::BLK) {
        fold();
        float v[C::BLK][CPL], P[C::BLK][CPL], gv[C::BLK][CPL];
        bool fast = true;
        {
          float nc[CPL];
#pragma unroll
          for (int q = 0; q < CPL; ++q) nc[q] = 0.f;
#pragma unroll
          for (int s = 0; s < C::BLK; ++s) {
            float dv[CPL], xv[CPL];
            const uint32_t ro = (r0 + s) * CPW * es;
            ChanLd<TI, CPL>::ld(td + ro, dv);
            ChanLd<TI, CPL>::ld(tx + ro, xv);
            ChanLd<TI, CPL>::ld(tg + ro, gv[s]);
#pragma unroll
            for (int q = 0; q < CPL; ++q) {
              nc[q] = fmaf(-A2[q], dv[q], nc[q]);
              v[s][q] = dv[q] * xv[q] * ex2_approx(nc[q]);
              P[s][q] = ex2_approx(-nc[q]);
            }
          }
#pragma unroll
          for (int q = 0; q < CPL; ++q) {
            fast = fast && nc[q] <= 60.f;
            ncl[q] = nc[q];
          }
        }
        if (__all_sync(0xffffffffu, fast)) {
          float4 bq[2][NQ], cq[2][NQ];
          if (kPrefetch) load_bc(tbc + r0 * 2 * N * 4, bq[0], cq[0]);
#pragma unroll
          for (int s = 0; s < C::BLK; ++s) {
            float y[CPL], o[CPL];
            if (kPrefetch) {
              if (s + 1 < C::BLK) load_bc(tbc + (r0 + s + 1) * 2 * N * 4, bq[(s + 1) & 1], cq[(s + 1) & 1]);
            } else {
              load_bc(tbc + (r0 + s) * 2 * N * 4, bq[s & 1], cq[s & 1]);
            }
            const float cb = __shfl_sync(0xffffffffu, cb_row, (r0 + s) * C::LPR);
            step_core(bq[s & 1], cq[s & 1], v[s], cb, y);
#pragma unroll
            for (int q = 0; q < CPL; ++q) o[q] = gv[s][q] * P[s][q] * y[q];
            if (ywriter) ChanLd<TI, CPL>::st(yt + ((r0 + s) * CPW + ccol) * es, o);
          }
        } else {
#pragma unroll
          for (int q = 0; q < CPL; ++q) ncl[q] = 0.f;
          float unused[CPL];
#pragma unroll 1
          for (int s = 0; s < C::BLK; ++s) {
            float dv[CPL], xv[CPL], gt[CPL], vv[CPL], y[CPL], o[CPL];
            const uint32_t ro = (r0 + s) * CPW * es;
            ChanLd<TI, CPL>::ld(td + ro, dv);
            ChanLd<TI, CPL>::ld(tx + ro, xv);
            ChanLd<TI, CPL>::ld(tg + ro, gt);
            slow_scalars(dv, xv, vv, unused);
            float4 bq[NQ], cq[NQ];
            load_bc(tbc + (r0 + s) * 2 * N * 4, bq, cq);
            const float cb = __shfl_sync(0xffffffffu, cb_row, (r0 + s) * C::LPR);
            step_core(bq, cq, vv, cb, y);
#pragma unroll
            for (int q = 0; q < CPL; ++q) o[q] = gt[q] * ex2_approx(-ncl[q]) * y[q];
            if (ywriter) ChanLd<TI, CPL>::st(yt + ((r0 + s) * CPW + ccol) * es, o);
          }
        }
      }
      // every lane is done with the slot and the y tile: refill the slot, store y
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (k + C::STAGES < k_end) issue(k + C::STAGES, true);
        tma_store_3d(&tmY, yt, wcol, p.t0 + k * C::ROWS, b);
        bulk_commit();
      }
    }
  }
  // state after the last row: the last chunk's warp, h = P g with -log2 P = ncl (rows past
  // T loaded as zeros leave it unchanged)
  if (p.h_out && active && ok && chunk == sp.S - 1) {
#pragma unroll
    for (int q = 0; q < CPL; ++q) {
      if (c0 + q < p.Di) {
        const float P = ex2_approx(-ncl[q]);
        float* ho = p.h_out + (static_cast<long long>(b) * p.Di + c0 + q) * N + n0;
#pragma unroll
        for (int j = 0; j < NQ; ++j) {   // undo the rotated chunk order (see g0 above)
          const int e = ((j + rot) & (NQ - 1)) * 4;
          ho[e] = g[q][2 * j].x * P;
          ho[e + 1] = g[q][2 * j].y * P;
          ho[e + 2] = g[q][2 * j + 1].x * P;
          ho[e + 3] = g[q][2 * j + 1].y * P;
        }
      }
    }
  }
  if (lane == 0) {
    bulk_wait_all();
    if (!ok) {  // let the copies this warp issued but did not consume land before it exits
      int never = 0;
      for (uint32_t j = consumed; j < issued; ++j)
        mbar_wait(&full[j % C::STAGES], (j / C::STAGES) & 1u, nullptr, &never, 100000000ull);
    }
  }
}

// Per-state decay, A[c, n] = -exp(a_log[c, n]): the recurrence with one exp2 per state
// and step (the block forms above need one decay per channel).  TPC = N / NS lanes share
// a channel, each holding NS of its states; C_t . h_t is summed over those lanes by
// shuffles.  One pass over T per channel.
template <typename TI, int N>
__global__ void __launch_bounds__(128) scan_ps_kernel(const ScanParams p) {
  pdl_trigger();
  pdl_wait();
  constexpr int NS = N < 8 ? N : 8;
  constexpr int TPC = N / NS;          // lanes per channel
  constexpr int CPW = 32 / TPC;        // channels per warp
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ch = lane / TPC, slice = lane % TPC;
  const int c = (blockIdx.x * 4 + warp) * CPW + ch;
  const int b = blockIdx.y;
  const bool valid = c < p.Di;
  const int cc = valid ? c : 0;
  const int n0 = slice * NS;
  float A2[NS], h[NS];
#pragma unroll
  load_h0(p, b, cc, n0, NS, h);
#pragma unroll
  for (int n = 0; n < NS; ++n) A2[n] = -expf(p.a_log[static_cast<long long>(cc) * N + n0 + n]) * 1.4426950408889634f;
  const long long row0 = static_cast<long long>(b) * p.T;
  const TI* xp = static_cast<const TI*>(p.x) + row0 * p.Di + cc;
  const TI* dp = static_cast<const TI*>(p.dt) + row0 * p.Di + cc;
  const TI* gp = static_cast<const TI*>(p.gate) + row0 * p.Di + cc;
  const float* bp = p.bc + row0 * 2 * N + n0;
  TI* yp = static_cast<TI*>(p.y) + row0 * p.y_ld + cc;
#pragma unroll 1
  for (int t = p.t0; t < p.T; ++t) {
    const float d = to_f<TI>(dp[static_cast<long long>(t) * p.Di]);
    const float u = d * to_f<TI>(xp[static_cast<long long>(t) * p.Di]);
    const float* brow = bp + static_cast<long long>(t) * 2 * N;
    float y = 0.f;
#pragma unroll
    for (int j = 0; j < NS; j += 4) {
      const float4 bb = __ldg(reinterpret_cast<const float4*>(brow + j));
      const float4 cq = __ldg(reinterpret_cast<const float4*>(brow + N + j));
      const float bv[4] = {bb.x, bb.y, bb.z, bb.w}, cv[4] = {cq.x, cq.y, cq.z, cq.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        h[j + e] = fmaf(ex2_approx(A2[j + e] * d), h[j + e], u * bv[e]);
        y = fmaf(cv[e], h[j + e], y);
      }
    }
#pragma unroll
    for (int off = 1; off < TPC; off <<= 1) y += __shfl_xor_sync(0xffffffffu, y, off);
    if (valid && slice == 0)
      yp[static_cast<long long>(t) * p.y_ld] = from_f<TI>(to_f<TI>(gp[static_cast<long long>(t) * p.Di]) * y);
  }
  if (p.h_out && valid) {
    float* ho = p.h_out + (static_cast<long long>(b) * p.Di + c) * N + n0;
#pragma unroll
    for (int n = 0; n < NS; ++n) ho[n] = h[n];
  }
}

template <typename TI, int N>
cudaError_t launch_ps(const ScanDesc& s, cudaStream_t st) {
  constexpr int NS = N < 8 ? N : 8;
  constexpr int CPB = 4 * (32 / (N / NS));  // channels per block
  ScanParams p{s.x, s.dt, s.bc, s.gate, s.a_log, s.y, s.y_ld, s.T, s.d_inner, s.d_state, s.h_out, s.t0, s.h0,
               s.h0_bstride};
  dim3 grid((s.d_inner + CPB - 1) / CPB, s.batch);
  return launch(scan_ps_kernel<TI, N>, grid, dim3(128), 0, st, p);
}

template <typename TI>
cudaError_t launch_ps_t(const ScanDesc& s, cudaStream_t st) {
  switch (s.d_state) {
    case 16: return launch_ps<TI, 16>(s, st);
    case 32: return launch_ps<TI, 32>(s, st);
    case 64: return launch_ps<TI, 64>(s, st);
    case 128: return launch_ps<TI, 128>(s, st);
    case 256: return launch_ps<TI, 256>(s, st);
    default: return cudaErrorInvalidValue;
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

template <typename TI, int N, int TPC, int CPL>
cudaError_t launch_w(const ScanDesc& s, cudaStream_t st) {
  using C = WCfg<TI, N, TPC, CPL>;
  static_assert(C::CPW * sizeof(TI) % 16 == 0, "tile rows must be whole 16-byte units");
  const bool f32 = sizeof(TI) == 4;
  CUtensorMap tx, td, tg, tb, ty;
  if (!map3d(&tx, s.x, f32, s.batch, s.T, s.d_inner, s.d_inner, C::CPW, C::ROWS) ||
      !map3d(&td, s.dt, f32, s.batch, s.T, s.d_inner, s.d_inner, C::CPW, C::ROWS) ||
      !map3d(&tg, s.gate, f32, s.batch, s.T, s.d_inner, s.d_inner, C::CPW, C::ROWS) ||
      !map3d(&tb, s.bc, true, s.batch, s.T, 2 * N, 2 * N, 2 * N, C::ROWS) ||
      !map3d(&ty, s.y, f32, s.batch, s.T, s.d_inner, s.y_ld, C::CPW, C::ROWS))
    return cudaErrorInvalidValue;
  const int groups = (s.d_inner + C::CPW - 1) / C::CPW;
  const int n_tiles = (s.T - s.t0 + C::ROWS - 1) / C::ROWS;
  const int max_warps = (227 * 1024 - 128) / C::WARP_B < C::MAX_WARPS ? (227 * 1024 - 128) / C::WARP_B : C::MAX_WARPS;
  static std::atomic<uint64_t> attr_done{0};
  if (cudaError_t e = smem_attr_once(scan_w_kernel<TI, N, TPC, CPL>, max_warps * C::WARP_B + 128, attr_done))
    return e;
  // Time chunks S: the smallest split that gives about two warps per SM sub-partition,
  // else the largest whose grid still fits in one wave; chunks of at least 8 tiles.
  SplitParams sp{1, 4, n_tiles};
  for (int S = 1; S <= C::MAX_WARPS; S *= 2) {
    const int G = S >= 4 ? 1 : 4 / S, warps = G * S;
    if (warps > max_warps || (S > 1 && n_tiles < 8 * S)) break;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, scan_w_kernel<TI, N, TPC, CPL>, 32 * warps,
                                                      warps * C::WARP_B + 128) != cudaSuccess)
      per_sm = 0;
    const long long ctas = static_cast<long long>((groups + G - 1) / G) * s.batch;
    if (S > 1 && ctas > static_cast<long long>(per_sm) * num_sms()) break;
    sp = SplitParams{S, G, (n_tiles + S - 1) / S};
    if (ctas * warps >= 2LL * 4 * num_sms()) break;
  }
  const int warps = sp.G * sp.S;
  const int smem = warps * C::WARP_B + 128;
  ScanParams p{s.x, s.dt, s.bc, s.gate, s.a_log, s.y, s.y_ld, s.T, s.d_inner, s.d_state, s.h_out, s.t0, s.h0,
               s.h0_bstride};
  dim3 grid((groups + sp.G - 1) / sp.G, s.batch);
  return launch(scan_w_kernel<TI, N, TPC, CPL>, grid, dim3(32 * warps), smem, st, tx, td, tg, tb, ty, p, sp, s.status);
}

template <typename TI, int NS, int TPC, int NWT>
cudaError_t launch_one(const ScanDesc& s, cudaStream_t st) {
  constexpr int CPW = 32 / TPC;
  ScanParams p{s.x, s.dt, s.bc, s.gate, s.a_log, s.y, s.y_ld, s.T, s.d_inner, s.d_state, s.h_out, s.t0, s.h0,
               s.h0_bstride};
  dim3 grid((s.d_inner + CPW - 1) / CPW, s.batch);
  return launch(scan_kernel<TI, NS, TPC, NWT>, grid, dim3(32 * NWT), 0, st, p);
}

template <typename TI>
cudaError_t launch_t(const ScanDesc& s, cudaStream_t st) {
  // The TMA-staged single-pass kernel needs 16-byte aligned bases and row strides for
  // x, dt, gate, B|C and y; otherwise the per-channel kernel runs.
  auto a16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  const long long es = static_cast<long long>(sizeof(TI));
  const bool tma_ok = (s.d_inner * es) % 16 == 0 && (s.y_ld * es) % 16 == 0 && a16(s.x) && a16(s.dt) &&
                     a16(s.gate) && a16(s.bc) && a16(s.y);
  // a fused dt projection (dt_low set) exists only in the tensor-core kernels
  if (s.dt_low) return tma_ok && sizeof(TI) == 2 ? launch_scan_tc(s, st) : cudaErrorInvalidValue;
  if (tma_ok) {
#if HY_SCAN_TC
    if (sizeof(TI) == 2 && s.d_state == 16) {
      const cudaError_t e = launch_scan_tc(s, st);
      if (e != cudaErrorNotSupported) return e;
    }
#endif
    switch (s.d_state) {
      case 16: return launch_w<TI, 16, HY_SCAN16_TPC, HY_SCAN16_CPL>(s, st);
      case 32: return launch_w<TI, 32, 1, 1>(s, st);
      case 64: return launch_w<TI, 64, 4, 2>(s, st);
      case 128: return launch_w<TI, 128, HY_SCAN128_TPC, HY_SCAN128_CPL>(s, st);
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
  if (s.a_per_state) {
    if (s.dt_low) return cudaErrorNotSupported;  // the fused dt projection is the block form's
    return s.bf16 ? launch_ps_t<__nv_bfloat16>(s, st) : launch_ps_t<float>(s, st);
  }
  return s.bf16 ? launch_t<__nv_bfloat16>(s, st) : launch_t<float>(s, st);
}

}  // namespace hy
