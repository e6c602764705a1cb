// scan_tc.cu -- the selective scan of the SSM heads as block matrix products on the
// 5th-generation tensor cores (bf16 layers, d_state = 16).
//
// Hymba writes its SSM head as a mixing matrix (blog.outta.ai Hymba review, "Design
// formulation"): y_i = G_i . sum_{j<=i} alpha_ij x_j with
//   alpha_ij = C_i (prod_{k=j+1..i} exp(A dt_k)) B_j dt_j.
// With A one scalar per channel the decay product factors: write
// lambda_t = sum_{k<=t} |A| dt_k / ln 2 within a block of Q = 64 steps and a reference
// r (the block's lambda after its first 32 steps).  Then for s <= t in the block
//   prod_{k=s+1..t} exp(A dt_k) = 2^(r - lambda_t) * 2^(lambda_s - r)
// and the block's output is, per channel c (h_in the state entering the block),
//   y[c,t] = W[c,t] * ( sum_s V[c,s] M[t,s] + sum_n G'[c,n] C[t,n] )
//   V[c,s] = dt x 2^(lambda_s - r),  W[c,t] = gate 2^(r - lambda_t),
//   M[t,s] = (C_t . B_s) [s <= t],   G'[c,n] = h_in[c,n] 2^(-r).
// The state leaving the block is h_out = 2^(-lambda_63) h_in + 2^(r - lambda_63) V B.
// So each block is four small tensor-core products that every channel shares the
// operands of: M = C B^T (once per block for all channels), Y = V M^T + G' C^T, and
// dG = V B.  Only the prefix sums, the exponentials and the 16-element state update
// per channel and block run on the CUDA cores.
//
// Ranges: |lambda_s - r| stays below 2^100 when both half-block decay sums stay
// below 100 (log2 units), which keeps every factor a normal fp32 number.  A block
// where some channel of the CTA exceeds that (very large dt) is run on the CUDA
// cores by the plain recurrence instead, for every channel of the CTA.
//
// dt itself can come in two ways: read from memory, or computed here from the
// low-rank projection (the layer's dt_proj, softplus(dt_low W_dt^T + b_dt)) as a fifth
// product per block, W_dt[c,:] . dt_low[t,:] with the CTA's 128 rows of W_dt resident
// in shared memory, so dt never goes through HBM.
//
// CTA = 128 channels of one sequence, all T steps, 384 threads:
//   warps 0-7   channel warps: warp w owns TMEM lane quadrant w % 4 (channel
//               32 (w % 4) + lane) and half w / 4 of each block's 64 steps; half 1
//               also carries the state chain and the large-decay path.
//   warps 8-9   mask C B^T (TMEM lanes 0-63 = t) into M, transpose B into B^T.
//   warp 10     TMA producer (x, dt, gate [64 t][128 c] bf16 or dt_low [64 t][64] bf16;
//               B|C [64 t][32] fp32).
//   warp 11     TMEM owner and MMA issuer.
// Operands: V, G' in TMEM (A from TMEM); M, B^T, C in shared memory, 128-byte
// swizzled K-major; accumulators Y (64 columns), dG (16), C B^T (64), W_dt dt_low^T (64)
// in TMEM; the scan's products kind::tf32, the dt projection kind::f16 (bf16), all with
// fp32 accumulation.  y goes out through a double-buffered shared tile and TMA stores.
#include "hy_common.cuh"
#include "hy_kernels.h"

namespace hy {
namespace {

constexpr int Q = 64;         // steps per block
constexpr int CH = 128;       // channels per CTA (TMEM lanes)
constexpr int NST = 16;       // state size handled here
constexpr int STAGES = 3;
constexpr int NTHR = 384;
constexpr int NCHT = 256;     // channel threads (named barrier 1)
constexpr float kRange = 100.f;  // max half-block decay sum (log2 units) for the product form

constexpr int TILE_B = Q * CH * 2;       // [64 t][128 c] bf16
constexpr int BC_B = Q * 2 * NST * 4;    // [64 t][B 16 | C 16] fp32, 128-byte rows
constexpr int MT_B = Q * Q * 4;          // M [t][s] tf32: two K chunks of [64 rows][128 B]
constexpr int BT_B = NST * Q * 4;        // B^T [n][s] tf32: two K chunks of [16 rows][128 B]
constexpr int KR = 64;                   // dt_rank capacity of the fused dt projection
constexpr int DL_B = Q * KR * 2;         // dt_low [64 t][64 r] bf16, 128-byte swizzle
constexpr int WD_B = CH * KR * 2;        // W_dt rows of the CTA [128 c][64 r] bf16, 128-byte swizzle

// Shared-memory layout (offsets from a 1024-aligned base).  Stage s holds x, gate, the
// dt tile (dt, or dt_low when FUSED) and B|C of one 64-step block.
template <bool FUSED>
struct Lay {
  static constexpr int D_B = FUSED ? DL_B : TILE_B;
  static constexpr int OFF_X = 0;
  static constexpr int OFF_G = OFF_X + STAGES * TILE_B;
  static constexpr int OFF_BC = OFF_G + STAGES * TILE_B;
  static constexpr int OFF_MT = OFF_BC + STAGES * BC_B;   // also the rows C B^T reads past the last B|C tile
  static constexpr int OFF_BT = OFF_MT + MT_B;
  static constexpr int OFF_D = OFF_BT + BT_B;
  static constexpr int OFF_WD = OFF_D + STAGES * D_B;     // FUSED only
  static constexpr int OFF_Y = OFF_WD + (FUSED ? WD_B : 0);
  static constexpr int OFF_S = OFF_Y + 2 * TILE_B;        // float [2][128]: half-block decay sums
  static constexpr int OFF_BAR = OFF_S + 2 * CH * 4;
  static constexpr int NBAR = 2 * STAGES + 4 * 2 + 4;
  static constexpr int SMEM_TOTAL = OFF_BAR + NBAR * 8 + 16 + 1024;  // + alignment of the base
  static_assert(OFF_BC % 1024 == 0 && OFF_MT % 1024 == 0 && OFF_BT % 1024 == 0 && OFF_D % 1024 == 0 &&
                    OFF_WD % 1024 == 0 && D_B % 1024 == 0,
                "swizzled tiles 1024-aligned");
  static_assert(SMEM_TOTAL <= 227 * 1024, "shared memory");
};

// TMEM columns (512 allocated)
constexpr uint32_t COL_Y = 0;      // [2][64]
constexpr uint32_t COL_W = 128;    // [2][64]; dt of a block that runs the plain recurrence
constexpr uint32_t COL_V = 256;    // [64]
constexpr uint32_t COL_DT = 320;   // [64]: W_dt dt_low^T (FUSED)
constexpr uint32_t COL_MR = 384;   // [64]: C B^T (lanes 0-63)
constexpr uint32_t COL_DG = 448;   // [2][16]
constexpr uint32_t COL_GP = 480;   // [2][16]
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t IDESC_N64 = idesc_tf32(128, 64);
constexpr uint32_t IDESC_N16 = idesc_tf32(128, 16);
constexpr uint32_t IDESC_DT = idesc_bf16(128, 64, false, false);

HY_DEV float bf2f(uint16_t u) { return __uint_as_float(static_cast<uint32_t>(u) << 16); }
// fp32 -> tf32 bit pattern, magnitude rounded to nearest (ties away from zero), on the
// integer pipe: add half of the dropped 13-bit field and clear it.
HY_DEV uint32_t tf32_round(float x) { return (__float_as_uint(x) + 0x1000u) & 0xFFFFE000u; }
// Two lanes of softplus(z) = max(z, 0) + log1p(e^-|z|), the log1p as u q(u) with the
// same degree-5 polynomial as softplus_f, on paired fp32 operations.
HY_DEV float2 softplus2(float2 z) {
  const float2 a = __fmul2_rn(make_float2(fabsf(z.x), fabsf(z.y)),
                              make_float2(-1.4426950408889634f, -1.4426950408889634f));
  const float2 u = make_float2(ex2_approx(a.x), ex2_approx(a.y));
  float2 q = __ffma2_rn(make_float2(-0.02386615f, -0.02386615f), u, make_float2(0.10121477f, 0.10121477f));
  q = __ffma2_rn(q, u, make_float2(-0.21004209f, -0.21004209f));
  q = __ffma2_rn(q, u, make_float2(0.32520431f, 0.32520431f));
  q = __ffma2_rn(q, u, make_float2(-0.49936107f, -0.49936107f));
  q = __ffma2_rn(q, u, make_float2(0.99999160f, 0.99999160f));
  return __ffma2_rn(u, q, make_float2(fmaxf(z.x, 0.f), fmaxf(z.y, 0.f)));
}

template <bool FUSED>
__global__ void __launch_bounds__(NTHR, 1)
    scan_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmD,
                   const __grid_constant__ CUtensorMap tmG, const __grid_constant__ CUtensorMap tmBC,
                   const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmWD,
                   const float* __restrict__ a_log, const float* __restrict__ b_dt, int T, int Di,
                   float* __restrict__ h_out, int t0, const float* __restrict__ h0, long long h0_bstride,
                   unsigned* status) {
  using L = Lay<FUSED>;
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);
  uint64_t* full = bars;                    // [STAGES] TMA landed
  uint64_t* empty = full + STAGES;          // [STAGES] last MMA reading the stage done
  uint64_t* vready = empty + STAGES;        // [2] V, W in TMEM (256 arrivals)
  uint64_t* dgready = vready + 2;           // [2] Y = V M^T and dG = V B done (V free)
  uint64_t* gready = dgready + 2;           // [2] G' in TMEM (128 arrivals)
  uint64_t* yready = gready + 2;            // [2] Y complete
  uint64_t* mraw = yready + 2;              // C B^T in TMEM
  uint64_t* mready = mraw + 1;              // M and B^T in shared memory (64 arrivals)
  uint64_t* dtready = mready + 1;           // W_dt dt_low^T in TMEM (FUSED)
  uint64_t* mma_done = dtready + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* sS = reinterpret_cast<float*>(sm + L::OFF_S);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c0 = blockIdx.x * CH, b = blockIdx.y;
  const int nblk = (T - t0 + Q - 1) / Q;   // blocks of rows [t0, T)

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&vready[i], NCHT);
      mbar_init(&dgready[i], 1);
      mbar_init(&gready[i], NCHT / 2);
      mbar_init(&yready[i], 1);
    }
    mbar_init(mraw, 1);
    mbar_init(mready, 64);
    mbar_init(dtready, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 11) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  pdl_wait();
  if (threadIdx.x == 320) {
    tma_prefetch(&tmX);
    tma_prefetch(&tmD);
    tma_prefetch(&tmG);
    tma_prefetch(&tmBC);
    tma_prefetch(&tmY);
    if (FUSED) tma_prefetch(&tmWD);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(sm);

  if (warp == 10) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int k = 0;
      for (; k < nblk; ++k) {
        const int s = k % STAGES;
        if (k >= STAGES && !mbar_wait(&empty[s], ((k / STAGES) - 1) & 1u, status, abort_flag)) break;
        mbar_arrive_expect_tx(&full[s], 2 * TILE_B + L::D_B + BC_B + (FUSED && k == 0 ? WD_B : 0));
        if (FUSED && k == 0) tma_load_2d(sm + L::OFF_WD, &tmWD, &full[s], 0, c0);
        tma_load_3d(sm + L::OFF_X + s * TILE_B, &tmX, &full[s], c0, t0 + k * Q, b);
        tma_load_3d(sm + L::OFF_D + s * L::D_B, &tmD, &full[s], FUSED ? 0 : c0, t0 + k * Q, b);
        tma_load_3d(sm + L::OFF_G + s * TILE_B, &tmG, &full[s], c0, t0 + k * Q, b);
        tma_load_3d(sm + L::OFF_BC + s * BC_B, &tmBC, &full[s], 0, t0 + k * Q, b);
      }
      if (k < nblk) {  // aborted: let the copies already issued land before smem goes away
        int never = 0;
        for (int j = (k > STAGES ? k - STAGES : 0); j < k; ++j)
          mbar_wait(&full[j % STAGES], (j / STAGES) & 1u, nullptr, &never, 100000000ull);
      }
    }
  } else if (warp == 11) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // descriptors of the first stage's tiles; every other tile is a fixed offset away
      const uint64_t dMT = sdesc_sw128(sbase + L::OFF_MT, 16, 1024), dBT = sdesc_sw128(sbase + L::OFF_BT, 16, 1024),
                     dBC = sdesc_sw128(sbase + L::OFF_BC, 16, 1024), dD = sdesc_sw128(sbase + L::OFF_D, 16, 1024),
                     dWD = sdesc_sw128(sbase + L::OFF_WD, 16, 1024);
      // Block k's stage has landed: W_dt dt_low^T (FUSED) and C B^T.
      auto issue_stage = [&](int k) -> bool {
        const int s = k % STAGES;
        if (!mbar_wait(&full[s], (k / STAGES) & 1u, status, abort_flag)) return false;
        tc_fence_after();
        if (FUSED) {
          const uint64_t dl = sdesc_add(dD, s * L::D_B);
#pragma unroll
          for (int j = 0; j < KR / 16; ++j)
            umma_bf16_ss(tmem + COL_DT, sdesc_add(dWD, 32 * j), sdesc_add(dl, 32 * j), IDESC_DT, j);
          umma_commit(dtready);
        }
        const uint64_t bc = sdesc_add(dBC, s * BC_B);
        // C B^T: A = C rows (128 rows read; rows 64..127 are whatever follows the tile and
        // land in TMEM lanes nobody reads), B = B rows; K = 16 = two tf32 steps.
#pragma unroll
        for (int j = 0; j < 2; ++j)
          umma_tf32_ss(tmem + COL_MR, sdesc_add(bc, 64 + 32 * j), sdesc_add(bc, 32 * j), IDESC_N64, j);
        umma_commit(mraw);
        return true;
      };
      bool ok = nblk > 0 && issue_stage(0);
      for (int k = 0; ok && k < nblk; ++k) {
        const int i = k & 1, s = k % STAGES;
        const uint32_t par = (k >> 1) & 1u;
        if (!mbar_wait(&vready[i], par, status, abort_flag) || !mbar_wait(mready, k & 1u, status, abort_flag)) break;
        tc_fence_after();
        // Y = V M^T (K = s, 64 = 8 steps) and dG = V B (B^T tile)
#pragma unroll
        for (int j = 0; j < 8; ++j)
          umma_tf32_ts(tmem + COL_Y + 64 * i, tmem + COL_V + 8 * j, sdesc_add(dMT, (j >> 2) * 8192 + (j & 3) * 32),
                       IDESC_N64, j);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          umma_tf32_ts(tmem + COL_DG + 16 * i, tmem + COL_V + 8 * j, sdesc_add(dBT, (j >> 2) * 2048 + (j & 3) * 32),
                       IDESC_N16, j);
        umma_commit(&dgready[i]);
        // the next block's dt projection and C B^T (their TMEM was read before vready / mready)
        if (k + 1 < nblk && !issue_stage(k + 1)) break;
        if (!mbar_wait(&gready[i], par, status, abort_flag)) break;
        tc_fence_after();
        // Y += G' C^T (K = n = 16)
        const uint64_t bc = sdesc_add(dBC, s * BC_B);
#pragma unroll
        for (int j = 0; j < 2; ++j)
          umma_tf32_ts(tmem + COL_Y + 64 * i, tmem + COL_GP + 16 * i + 8 * j, sdesc_add(bc, 64 + 32 * j), IDESC_N64, 1);
        umma_commit(&yready[i]);
        umma_commit(&empty[s]);
      }
      umma_commit(mma_done);
      int never = 0;
      mbar_wait(mma_done, 0, nullptr, &never, 100000000ull);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ M = mask(C B^T), B^T
    const int t = (warp - 8) * 32 + lane;  // TMEM lane = step within the block
    const uint32_t tl = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    uint8_t* mt = sm + L::OFF_MT;
    uint8_t* bt = sm + L::OFF_BT;
    for (int k = 0; k < nblk; ++k) {
      const int s = k % STAGES;
      bool ok = mbar_wait(mraw, k & 1u, status, abort_flag) && mbar_wait(&full[s], (k / STAGES) & 1u, status, abort_flag);
      if (ok && k > 0) ok = mbar_wait(&dgready[(k - 1) & 1], ((k - 1) >> 1) & 1u, status, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t r[2][32];
      tmem_ld32(tl + COL_MR, r[0]);
      tmem_ld32(tl + COL_MR + 32, r[1]);
      tmem_wait_ld();
      // row t of M (K-major, 128-byte swizzle): s in [32 h, 32 h + 32) -> chunk h
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint8_t* row = mt + h * 8192 + (t >> 3) * 1024 + (t & 7) * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint32_t v[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int si = 32 * h + 4 * j + e;
            v[e] = si <= t ? tf32_round(__uint_as_float(r[h][4 * j + e])) : 0u;
          }
          *reinterpret_cast<uint4*>(row + ((j ^ (t & 7)) << 4)) = make_uint4(v[0], v[1], v[2], v[3]);
        }
      }
      // B^T [n][s]: element (n, s = t)
      const uint8_t* bcrow = sm + L::OFF_BC + s * BC_B + t * 128;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 q = *reinterpret_cast<const float4*>(bcrow + ((j ^ (t & 7)) << 4));
        const float qv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int n = 4 * j + e;
          uint8_t* dst = bt + (t >> 5) * 2048 + (n >> 3) * 1024 + (n & 7) * 128 + ((((t & 31) >> 2) ^ (n & 7)) << 4) +
                         (t & 3) * 4;
          *reinterpret_cast<uint32_t*>(dst) = tf32_round(qv[e]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(mready);
    }
  } else {
    // ------------------------------------------------------------ channel warps
    const int qd = warp & 3, half = warp >> 2;
    const int cl = qd * 32 + lane, c = c0 + cl;
    const uint32_t tl = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    const float A2 = c < Di ? expf(a_log[c]) * 1.4426950408889634f : 0.f;  // |A| / ln 2
    const float bdt = FUSED && c < Di ? b_dt[c] : 0.f;
    float h[NST];   // the state entering the current block (half 1), from h0 at row t0
#pragma unroll
    for (int n = 0; n < NST; ++n) h[n] = 0.f;
    if (h0 && c < Di) {
      const float4* hi = reinterpret_cast<const float4*>(h0 + b * h0_bstride + static_cast<long long>(c) * NST);
#pragma unroll
      for (int j = 0; j < NST / 4; ++j) {
        const float4 v = hi[j];
        h[4 * j] = v.x; h[4 * j + 1] = v.y; h[4 * j + 2] = v.z; h[4 * j + 3] = v.w;
      }
    }
    float pS0 = 0.f, pS1 = 0.f;  // previous block's half sums (chain)
    bool prev_any = false;
    for (int k = 0; k <= nblk; ++k) {
      bool fail = false;
      bool any = false;
      if (k < nblk) {
        const int s = k % STAGES, i = k & 1;
        const uint8_t* xt = sm + L::OFF_X + s * TILE_B + cl * 2;
        const uint8_t* gt = sm + L::OFF_G + s * TILE_B + cl * 2;
        fail = !__all_sync(0xffffffffu, mbar_wait(&full[s], (k / STAGES) & 1u, status, abort_flag));
        // ---- dt of this half block, and its decay sum
        float dtv[32];
        float2 S2 = make_float2(0.f, 0.f);
        if (FUSED) {
          if (!fail) fail = !__all_sync(0xffffffffu, mbar_wait(dtready, k & 1u, status, abort_flag));
          uint32_t z[32];
          if (!fail) {
            tc_fence_after();
            tmem_ld32(tl + COL_DT + 32 * half, z);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) z[j] = 0u;
          }
          // steps past T (zero-filled dt_low) get dt = 0, so they leave the state alone
          const int t_end = T - (t0 + k * Q + 32 * half);
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            float2 d = softplus2(make_float2(__uint_as_float(z[j]) + bdt, __uint_as_float(z[j + 1]) + bdt));
            if (j >= t_end) d.x = 0.f;
            if (j + 1 >= t_end) d.y = 0.f;
            dtv[j] = d.x;
            dtv[j + 1] = d.y;
            S2 = __ffma2_rn(make_float2(A2, A2), d, S2);
          }
        } else {
          const uint8_t* dtt = sm + L::OFF_D + s * L::D_B + cl * 2;
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            dtv[j] = bf2f(*reinterpret_cast<const uint16_t*>(dtt + (32 * half + j) * 256));
            dtv[j + 1] = bf2f(*reinterpret_cast<const uint16_t*>(dtt + (32 * half + j + 1) * 256));
            S2 = __ffma2_rn(make_float2(A2, A2), make_float2(dtv[j], dtv[j + 1]), S2);
          }
        }
        const float S = S2.x + S2.y;
        sS[half * CH + cl] = S;
        any = bar_red_or(1, NCHT, fail || !(S <= kRange));
        // ---- V = dt x 2^(lambda - r), W = gate 2^(r - lambda) into TMEM.  In a block that
        // runs the plain recurrence V is zero and the W columns carry dt instead.
        if (!fail) {
          uint32_t vr[32], wr[32];
          if (!any) {
            float mu = half ? 0.f : -S;  // lambda - r
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const float mu0 = fmaf(A2, dtv[j], mu);
              mu = fmaf(A2, dtv[j + 1], mu0);
              const int row = (32 * half + j) * 256;
              const float2 xv = make_float2(bf2f(*reinterpret_cast<const uint16_t*>(xt + row)),
                                            bf2f(*reinterpret_cast<const uint16_t*>(xt + row + 256)));
              const float2 gv = make_float2(bf2f(*reinterpret_cast<const uint16_t*>(gt + row)),
                                            bf2f(*reinterpret_cast<const uint16_t*>(gt + row + 256)));
              const float2 e = make_float2(ex2_approx(mu0), ex2_approx(mu));
              const float2 v = __fmul2_rn(__fmul2_rn(make_float2(dtv[j], dtv[j + 1]), xv), e);
              const float2 w = __fmul2_rn(gv, make_float2(ex2_approx(-mu0), ex2_approx(-mu)));
              vr[j] = tf32_round(v.x);
              vr[j + 1] = tf32_round(v.y);
              wr[j] = __float_as_uint(w.x);
              wr[j + 1] = __float_as_uint(w.y);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              vr[j] = 0u;
              wr[j] = __float_as_uint(dtv[j]);
            }
          }
          // V has one buffer: the products of block k - 1 must have read it
          if (k > 0) fail = !__all_sync(0xffffffffu, mbar_wait(&dgready[(k - 1) & 1], ((k - 1) >> 1) & 1u, status,
                                                                 abort_flag));
          if (!fail) {
            tc_fence_after();
            tmem_st32(tl + COL_V + 32 * half, vr);
            tmem_st32(tl + COL_W + 64 * i + 32 * half, wr);
            tmem_wait_st();
            tc_fence_before();
          }
        }
        mbar_arrive(&vready[i]);
        // ---- state chain: h entering block k, G' = h 2^(-r)  (half 1)
        if (half == 1 && !fail) {
          const float S0 = sS[cl], S1 = S;
          if (k > 0 && !prev_any) {  // dG of block k - 1 is complete (waited above)
            uint32_t d[16];
            tmem_ld16(tl + COL_DG + 16 * ((k - 1) & 1), d);
            tmem_wait_ld();
            const float a = ex2_approx(-(pS0 + pS1)), bs = ex2_approx(-pS1);
#pragma unroll
            for (int n = 0; n < NST; ++n) h[n] = fmaf(a, h[n], bs * __uint_as_float(d[n]));
          }
          uint32_t gp[16];
          const float sc = ex2_approx(-S0);
#pragma unroll
          for (int n = 0; n < NST; ++n) gp[n] = any ? 0u : tf32_round(h[n] * sc);
          tmem_st16(tl + COL_GP + 16 * i, gp);
          tmem_wait_st();
          tc_fence_before();
          pS0 = S0;
          pS1 = S1;
        }
        // ---- large decays: the plain recurrence over the block, y into the y tile.  G' is
        // announced only after it, since the MMA that waits for G' frees the stage.
        if (any) {
          if (threadIdx.x == 0) bulk_wait_all();  // the store that last read this y tile is done
          bar_sync_n(1, NCHT);                    // and every half's dt is in the W columns
          if (half == 1 && !fail) {
            tc_fence_after();
            uint8_t* yt = sm + L::OFF_Y + i * TILE_B + cl * 2;
            const uint8_t* bct = sm + L::OFF_BC + s * BC_B;
#pragma unroll 1
            for (int t0 = 0; t0 < Q; t0 += 16) {
              uint32_t dq[16];
              tmem_ld16(tl + COL_W + 64 * i + t0, dq);
              tmem_wait_ld();
#pragma unroll
              for (int tt = 0; tt < 16; ++tt) {
                const int t = t0 + tt;
                const float dt = __uint_as_float(dq[tt]);
                const float xv = bf2f(*reinterpret_cast<const uint16_t*>(xt + t * 256));
                const float gv = bf2f(*reinterpret_cast<const uint16_t*>(gt + t * 256));
                const float a = ex2_approx(-A2 * dt), u = dt * xv;
                const uint8_t* row = bct + t * 128;
                float y = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  const float4 bq = *reinterpret_cast<const float4*>(row + ((j ^ (t & 7)) << 4));
                  const float4 cq = *reinterpret_cast<const float4*>(row + (((j + 4) ^ (t & 7)) << 4));
                  h[4 * j + 0] = fmaf(a, h[4 * j + 0], u * bq.x);
                  h[4 * j + 1] = fmaf(a, h[4 * j + 1], u * bq.y);
                  h[4 * j + 2] = fmaf(a, h[4 * j + 2], u * bq.z);
                  h[4 * j + 3] = fmaf(a, h[4 * j + 3], u * bq.w);
                  y = fmaf(cq.x, h[4 * j + 0], y);
                  y = fmaf(cq.y, h[4 * j + 1], y);
                  y = fmaf(cq.z, h[4 * j + 2], y);
                  y = fmaf(cq.w, h[4 * j + 3], y);
                }
                *reinterpret_cast<uint16_t*>(yt + t * 256) = bf16_bits(gv * y);
              }
            }
          }
        }
        if (half == 1) mbar_arrive(&gready[i]);
      }
      // ---- output of block k - 1: y = W * Y into the y tile, TMA store
      if (k > 0) {
        const int jb = k - 1, i = jb & 1;
        // after the last block no barrier has followed thread 0's wait for the store that
        // last read this y tile: meet one
        if (k == nblk) bar_sync_n(1, NCHT);
        if (!fail) {
          fail = !__all_sync(0xffffffffu, mbar_wait(&yready[i], (jb >> 1) & 1u, status, abort_flag));
          if (!fail && !prev_any) {
            tc_fence_after();
            uint32_t yv[32], wv[32];
            tmem_ld32(tl + COL_Y + 64 * i + 32 * half, yv);
            tmem_ld32(tl + COL_W + 64 * i + 32 * half, wv);
            tmem_wait_ld();
            uint8_t* yt = sm + L::OFF_Y + i * TILE_B + cl * 2 + 32 * half * 256;
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const float2 o = __fmul2_rn(make_float2(__uint_as_float(yv[j]), __uint_as_float(yv[j + 1])),
                                          make_float2(__uint_as_float(wv[j]), __uint_as_float(wv[j + 1])));
              const uint32_t p2 = pack_bf16(o.x, o.y);
              *reinterpret_cast<uint16_t*>(yt + j * 256) = static_cast<uint16_t>(p2);
              *reinterpret_cast<uint16_t*>(yt + (j + 1) * 256) = static_cast<uint16_t>(p2 >> 16);
            }
          }
        }
        fence_proxy_async_smem();
        if (bar_red_or(1, NCHT, fail || *abort_flag)) break;
        if (threadIdx.x == 0) {
          tma_store_3d(&tmY, sm + L::OFF_Y + i * TILE_B, c0, t0 + jb * Q, b);
          bulk_commit();
          bulk_wait_read1();  // the store before it has read its tile: that tile may be rewritten
        }
      } else if (fail) {
        if (bar_red_or(1, NCHT, true)) break;
      } else {
        if (bar_red_or(1, NCHT, *abort_flag != 0)) break;
      }
      if (k < nblk) prev_any = any;
      if (k == nblk && h_out && half == 1) {  // warp-uniform (tcgen05.ld below is warp-collective)
        // state after the last row: h entering the last block advanced by that block's dG
        // (complete: its yready, waited above, was committed after it), unless the block
        // ran the plain recurrence, which left h there already
        if (!prev_any) {
          tc_fence_after();
          uint32_t d[16];
          tmem_ld16(tl + COL_DG + 16 * ((nblk - 1) & 1), d);
          tmem_wait_ld();
          const float a = ex2_approx(-(pS0 + pS1)), bs = ex2_approx(-pS1);
#pragma unroll
          for (int n = 0; n < NST; ++n) h[n] = fmaf(a, h[n], bs * __uint_as_float(d[n]));
        }
        if (c < Di) {
          float4* ho = reinterpret_cast<float4*>(h_out + (static_cast<long long>(b) * Di + c) * NST);
#pragma unroll
          for (int j = 0; j < NST / 4; ++j) ho[j] = make_float4(h[4 * j], h[4 * j + 1], h[4 * j + 2], h[4 * j + 3]);
        }
      }
    }
    if (threadIdx.x == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 11) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// 3-D map over [batch][T][cols] (row stride ld elements), box = bc x br x 1.
bool map3d(CUtensorMap* m, const void* base, bool f32, int batch, int T, long long cols, long long ld, int bc,
           int br, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const int es = f32 ? 4 : 2;
  cuuint64_t gd[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(batch)};
  cuuint64_t gs[2] = {static_cast<cuuint64_t>(ld) * es, static_cast<cuuint64_t>(ld) * es * T};
  cuuint32_t bx[3] = {static_cast<cuuint32_t>(bc), static_cast<cuuint32_t>(br), 1}, el[3] = {1, 1, 1};
  return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
            gd, gs, bx, el, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over [rows][cols] (row stride ld elements), box = bc x br, 128-byte swizzle.
bool map2d_sw128(CUtensorMap* m, const void* base, long long rows, long long cols, long long ld, int bc, int br) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t gs[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t bx[2] = {static_cast<cuuint32_t>(bc), static_cast<cuuint32_t>(br)}, el[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gd, gs, bx, el,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool a16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; }

// 3-D fp32 map over nrec records of rec_bytes, each [rows][cols] with row stride
// row_bytes; box = bc x br x 1, 128-byte swizzle.
bool map_rec_f32(CUtensorMap* m, const void* base, long long cols, long long rows, long long row_bytes, long long nrec,
                 long long rec_bytes, int bc, int br) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(nrec)};
  cuuint64_t gs[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rec_bytes)};
  cuuint32_t bx[3] = {static_cast<cuuint32_t>(bc), static_cast<cuuint32_t>(br), 1}, el[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), gd, gs, bx, el,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool FUSED>
cudaError_t launch_tc(const ScanDesc& s, cudaStream_t st) {
  using L = Lay<FUSED>;
  CUtensorMap tx, td, tg, tb, ty, tw;
  bool ok = map3d(&tx, s.x, false, s.batch, s.T, s.d_inner, s.d_inner, CH, Q, CU_TENSOR_MAP_SWIZZLE_NONE) &&
            map3d(&tg, s.gate, false, s.batch, s.T, s.d_inner, s.d_inner, CH, Q, CU_TENSOR_MAP_SWIZZLE_NONE) &&
            map3d(&tb, s.bc, true, s.batch, s.T, 2 * NST, 2 * NST, 2 * NST, Q, CU_TENSOR_MAP_SWIZZLE_128B) &&
            map3d(&ty, s.y, false, s.batch, s.T, s.d_inner, s.y_ld, CH, Q, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (FUSED) {
    // dt_low tiles [64 t][KR r] (columns past dt_rank read as zero) and the CTA's W_dt rows
    ok = ok && map3d(&td, s.dt_low, false, s.batch, s.T, s.dt_rank, s.dt_rank, KR, Q, CU_TENSOR_MAP_SWIZZLE_128B) &&
         map2d_sw128(&tw, s.w_dt, s.d_inner, s.dt_rank, s.dt_rank, KR, CH);
  } else {
    ok = ok && map3d(&td, s.dt, false, s.batch, s.T, s.d_inner, s.d_inner, CH, Q, CU_TENSOR_MAP_SWIZZLE_NONE);
    tw = tx;  // unused
  }
  if (!ok) return cudaErrorNotSupported;
  static std::atomic<uint64_t> attr_done{0};
  if (cudaError_t e = smem_attr_once(scan_tc_kernel<FUSED>, L::SMEM_TOTAL, attr_done)) return e;
  dim3 grid((s.d_inner + CH - 1) / CH, s.batch);
  return launch(scan_tc_kernel<FUSED>, grid, dim3(NTHR), L::SMEM_TOTAL, st, tx, td, tg, tb, ty, tw, s.a_log, s.b_dt,
                s.T, s.d_inner, s.h_out, s.t0, s.h0, s.h0_bstride, s.status);
}


// ---------------------------------------------------------------------------------
// d_state = 128.  The same block form, re-balanced for a state eight times larger.
//
// * The state lives in TMEM as G' (fp32, 128 columns), and the tensor core advances it
//   itself.  With r = S0 (the decay sum of a block's first half, log2 units) and S1 that
//   of its second half, the state leaving block k is h_{k+1} = 2^-S1 (G'_k + V_k B_k),
//   so G'_{k+1} = 2^-S0_{k+1} 2^-S1_k (G'_k + V_k B_k): the product dG = V B accumulates
//   straight into G' after Y = G' C^T has read it (tcgen05.mma of one thread execute in
//   issue order), and the CUDA cores rescale G' once per block, one multiply per element
//   (two factors, each at most 2^100, applied one after the other).
// * Blocks of Q = 32 steps (halves of 16): a B|C row is 1 KB, and two stages of 32 rows
//   of x, gate, dt_low and B|C (56 KB each) fit beside the other tiles.  B|C arrive as
//   eight 32-column boxes ([32 t][128 B] each, 128-byte swizzle): chunks 0-3 are B (n in
//   [32 q, 32 q + 32)), 4-7 are C, each one K atom of the tf32 products.
// * The per-block dependency chain is only: the state products of block k -> the state
//   warps rescale G' -> the state products of block k + 1.  Everything else is kept off
//   it: the copy warps turn each stage's B into B^T and copy C (both tf32, double-
//   buffered) as soon as it lands, so the stage is released long before the state
//   products read B and C; separate V/W warps form dt, the decay sums, V and W of the
//   blocks ahead (V, W triple-buffered in TMEM), so that the state warps only rescale G'
//   and write y; the part of Y that does not depend on the state (V M^T) is added after
//   the state products; and the MMA thread issues whichever of its four tasks is ready
//   (state products, a landed stage's dt projection and C B^T, V M^T, stage release)
//   instead of waiting in a fixed order.
// * The dt projection is always fused (dt_rank <= 128: one or two 64-column atoms of
//   dt_low and W_dt, columns past dt_rank zero-filled by TMA).
// * A block where some channel's half-block decay sum exceeds kRange runs the plain
//   recurrence on the CUDA cores (the half-1 state warps, 8 state columns at a time from
//   TMEM, B and C from the tf32 copies), with G' holding the raw state on exit; its V, W
//   columns then carry dt x and the gate, and the MMA thread skips its products.
// * y goes straight from registers to global memory (8-byte stores of 4 adjacent
//   channels after two shuffle rounds).
//
// CTA = 128 channels of one sequence, 640 threads: warps 0-7 state warps (TMEM quadrant
// w % 4, half w / 4 of G''s columns and of each block's output rows), warps 8-15 V/W
// warps (quadrant w % 4, half (w - 8) / 4 of each block's steps), warps 16-17 B^T and the
// C copy (warp 16 also the mask M, from TMEM lanes 0-31), warp 18 TMA, warp 19 TMEM and
// MMA.
namespace t128 {
constexpr int Q = 32;
constexpr int NS = 128;
constexpr int HQ = 16;                  // steps per V/W thread and block (a half)
constexpr int QQ = 8;                   // steps per pass of the plain recurrence
constexpr int NTHR2 = 608;
constexpr int NRT = 256;                // state threads
constexpr int NVT = 256;                // V/W threads (named barrier 1)
constexpr int KA = 64;                  // dt_rank per K atom of the dt projection
constexpr int TILE_B = Q * CH * 2;      // [32 t][128 c] bf16
constexpr int BCC_B = Q * 128;          // one 32-column chunk of C [32 t][32] fp32
constexpr int DLC_B = Q * 128;          // one dt_low atom [32 t][64 r] bf16 (of one stage)
constexpr int WDC_B = CH * 128;         // one W_dt atom [128 c][64 r] bf16
constexpr int MT_B = Q * Q * 4;         // M [t][s] tf32
constexpr int BT_B = NS * Q * 4;        // B^T [n][s] tf32
constexpr int CC_B = 4 * BCC_B;         // C [t][n] tf32, four chunks
constexpr int GREC_B = MT_B + BT_B + CC_B;  // a block's record from bc_gram_kernel
constexpr int ST = 4;                   // stages (x, gate, dt_low)
constexpr int OFF_DL = 0;
constexpr int OFF_WD = OFF_DL + 2 * ST * DLC_B;   // dt_low [atom][stage][32 t]: stages 2j, 2j + 1 adjacent
constexpr int OFF_MT = OFF_WD + 2 * WDC_B;
constexpr int OFF_BT = OFF_MT + 2 * MT_B;
constexpr int OFF_CC = OFF_BT + 2 * BT_B;
constexpr int OFF_X = OFF_CC + 2 * CC_B;
constexpr int OFF_G = OFF_X + ST * TILE_B;
constexpr int OFF_S = OFF_G + ST * TILE_B;   // float [2 blocks][2 halves][128]: half-block decay sums
constexpr int OFF_ANY = OFF_S + 2 * 2 * CH * 4;  // int [3]: the block runs the plain recurrence
constexpr int OFF_BAR = OFF_ANY + 16;
// full[ST] empty[ST] dtready[2] vready[3] btready[2] mready[2] gready dgready[2] yready[2] yidone wdone[3]
// mma_done
constexpr int NBAR = 2 * ST + 2 + 3 + 2 + 2 + 1 + 2 + 2 + 1 + 3 + 1;
constexpr int SMEM_TOTAL = OFF_BAR + NBAR * 8 + 16 + 1024;
static_assert(OFF_DL % 1024 == 0 && OFF_WD % 1024 == 0 && OFF_MT % 1024 == 0 && OFF_BT % 1024 == 0 &&
                  OFF_CC % 1024 == 0,
              "swizzled tiles 1024-aligned");
static_assert(SMEM_TOTAL <= 227 * 1024, "shared memory");

constexpr uint32_t COL_Y = 0;     // [2][32]
constexpr uint32_t COL_W = 64;    // [3][32]
constexpr uint32_t COL_V = 160;   // [3][32]
constexpr uint32_t COL_DT = 256;  // [4][32] W_dt dt_low^T (block k in slot k % 4)
constexpr uint32_t COL_GP = 384;  // [128] G'
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC_Q = idesc_tf32(128, Q);
constexpr uint32_t IDESC_N = idesc_tf32(128, NS);
constexpr uint32_t IDESC_DT = idesc_bf16(128, 2 * Q, false, false);   // two blocks at once

// Offsets of element (n, s) in B^T [n][s] and (t, n) in the C copy [t][n] (K-major,
// 128-byte swizzle; B^T one 128-row atom, C four 32-column chunks).
HY_DEV uint32_t bt_off(int n, int s) {
  return (n >> 3) * 1024 + (n & 7) * 128 + (((s >> 2) ^ (n & 7)) << 4) + (s & 3) * 4;
}
HY_DEV uint32_t cc_off(int t, int n) {
  return (n >> 5) * BCC_B + (t >> 3) * 1024 + (t & 7) * 128 + ((((n & 31) >> 2) ^ (t & 7)) << 4) + (n & 3) * 4;
}

// 8-column variants of the TMEM load and store (32 lanes x 8 consecutive 32-bit columns).
HY_DEV void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
HY_DEV void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// 16 consecutive rows (tb, tb + 1, ...) of y for this lane's channel, written as 8-byte
// stores of 4 adjacent channels: two shuffle rounds hand each lane 4 rows of its 4-lane
// group's channels (lane 4h + 2p + e ends with rows 4m + 2p + e, m < 4, channels 4h..4h+3),
// so a warp writes 4 x 8 rows x 64 bytes instead of 16 x 64-byte row pieces per thread.
// ybase: row 0, channel 0 of the sequence; c4: the group's first channel (a multiple of 4;
// d_inner is a multiple of 8, so a group is inside or outside d_inner as a whole).
HY_DEV void store_y16(__nv_bfloat16* ybase, long long y_ld, int tb, int T, int c4, bool c_ok, const float (&v)[16]) {
  const int lane = threadIdx.x & 31, e = lane & 1, p = (lane >> 1) & 1;
  uint32_t w[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) {  // rows 2m + e of channels (2 (lane >> 1), + 1)
    const float send = e ? v[2 * m] : v[2 * m + 1];
    const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
    w[m] = e ? pack_bf16(recv, v[2 * m + 1]) : pack_bf16(v[2 * m], recv);
  }
#pragma unroll
  for (int m = 0; m < 4; ++m) {  // rows 4m + 2p + e of channels c4 .. c4 + 3
    const uint32_t send = p ? w[2 * m] : w[2 * m + 1];
    const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, 2);
    const uint2 q = p ? make_uint2(recv, w[2 * m + 1]) : make_uint2(w[2 * m], recv);
    const int t = tb + 4 * m + 2 * p + e;
    if (c_ok && t < T) *reinterpret_cast<uint2*>(ybase + static_cast<long long>(t) * y_ld + c4) = q;
  }
}

// The operands every channel shares, once per block k (rows t0 + 32 k + t) of sequence
// b, into record b * nblk + k of GREC_B bytes (rows past T read as zero):
//   M   [t][s] = (C_t . B_s) [s <= t]: fp32 sums over n, rounded to tf32
//   B^T [n][s] = B_s[n], rounded to tf32
//   C   [t][n] = C_t[n], rounded to tf32
// each row-major, so that a 128-byte-swizzled TMA box lands in shared memory as the
// K-major operand of V M^T (M), of G' += V B (B^T) and of Y = G' C^T (C, four boxes of
// 32 columns).  One CTA per block.
__global__ void __launch_bounds__(256) bc_gram_kernel(const float* __restrict__ bc, int T, int t0, int nblk,
                                                      uint8_t* __restrict__ rec) {
  // no early trigger: the scan's CTAs (whose shared memory leaves no room for these)
  // start once every record is written
  __shared__ __align__(16) float sB[Q][NS + 4];   // rows padded by 16 bytes: conflict-free
  __shared__ __align__(16) float sC[Q][NS + 4];
  const int k = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int r0 = t0 + k * Q;
  pdl_wait();
  for (int i = tid; i < Q * 2 * NS / 4; i += blockDim.x) {  // a row: B 32 float4, C 32 float4
    const int r = i / (2 * NS / 4), q = i % (2 * NS / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + r < T) v = reinterpret_cast<const float4*>(bc + (static_cast<long long>(b) * T + r0 + r) * 2 * NS)[q];
    float* dst = q < NS / 4 ? &sB[r][4 * q] : &sC[r][4 * q - NS];
    *reinterpret_cast<float4*>(dst) = v;
  }
  __syncthreads();
  uint8_t* out = rec + (static_cast<long long>(b) * nblk + k) * GREC_B;
  if (tid < 64) {
    // M: thread = a 4 x 4 tile (rows t0..t0+3, columns s0..s0+3), paired FMAs along s
    const int t0 = (tid >> 3) * 4, s0 = (tid & 7) * 4;
    float2 acc[4][2];
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[r][0] = acc[r][1] = make_float2(0.f, 0.f);
#pragma unroll 2
    for (int n = 0; n < NS; n += 4) {
      float4 cv[4], bv[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        cv[r] = *reinterpret_cast<const float4*>(&sC[t0 + r][n]);
        bv[r] = *reinterpret_cast<const float4*>(&sB[s0 + r][n]);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float c4[4] = {cv[r].x, cv[r].y, cv[r].z, cv[r].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 cc = make_float2(c4[e], c4[e]);
          const float b0 = e == 0 ? bv[0].x : e == 1 ? bv[0].y : e == 2 ? bv[0].z : bv[0].w;
          const float b1 = e == 0 ? bv[1].x : e == 1 ? bv[1].y : e == 2 ? bv[1].z : bv[1].w;
          const float b2 = e == 0 ? bv[2].x : e == 1 ? bv[2].y : e == 2 ? bv[2].z : bv[2].w;
          const float b3 = e == 0 ? bv[3].x : e == 1 ? bv[3].y : e == 2 ? bv[3].z : bv[3].w;
          acc[r][0] = __ffma2_rn(cc, make_float2(b0, b1), acc[r][0]);
          acc[r][1] = __ffma2_rn(cc, make_float2(b2, b3), acc[r][1]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int t = t0 + r;
      uint4 o;
      o.x = s0 <= t ? tf32_round(acc[r][0].x) : 0u;
      o.y = s0 + 1 <= t ? tf32_round(acc[r][0].y) : 0u;
      o.z = s0 + 2 <= t ? tf32_round(acc[r][1].x) : 0u;
      o.w = s0 + 3 <= t ? tf32_round(acc[r][1].y) : 0u;
      reinterpret_cast<uint4*>(out)[t * (Q / 4) + s0 / 4] = o;
    }
  } else {
    // B^T (row n, columns 16 h .. 16 h + 15) and C (row t, columns 16 h .. 16 h + 15)
    for (int u = tid - 64; u < 2 * NS; u += 192) {
      const int n = u >> 1, h = u & 1;
      uint4* dst = reinterpret_cast<uint4*>(out + MT_B + n * Q * 4 + h * 64);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int s0 = 16 * h + 4 * j;
        dst[j] = make_uint4(tf32_round(sB[s0][n]), tf32_round(sB[s0 + 1][n]), tf32_round(sB[s0 + 2][n]),
                            tf32_round(sB[s0 + 3][n]));
      }
    }
    for (int u = tid - 64; u < Q * 8; u += 192) {
      const int t = u >> 3, h = u & 7;
      uint4* dst = reinterpret_cast<uint4*>(out + MT_B + BT_B + t * NS * 4 + h * 64);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 v = *reinterpret_cast<const float4*>(&sC[t][16 * h + 4 * j]);
        dst[j] = make_uint4(tf32_round(v.x), tf32_round(v.y), tf32_round(v.z), tf32_round(v.w));
      }
    }
  }
}

__global__ void __launch_bounds__(NTHR2, 1)
    scan_tc128_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmDL,
                      const __grid_constant__ CUtensorMap tmG, const __grid_constant__ CUtensorMap tmWD,
                      const __grid_constant__ CUtensorMap tmM, const __grid_constant__ CUtensorMap tmBT,
                      const __grid_constant__ CUtensorMap tmC,
                      const float* __restrict__ a_log, const float* __restrict__ b_dt, __nv_bfloat16* __restrict__ y,
                      long long y_ld, int T, int Di, int ka, float* __restrict__ h_out, int t0,
                      const float* __restrict__ h0, long long h0_bstride, unsigned* status) {
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + OFF_BAR);  // [ST] TMA landed
  uint64_t* empty = full + ST;         // [ST] the stage's x and gate read by the V/W warps (256 arrivals)
  uint64_t* dtready = empty + ST;      // [2] W_dt dt_low^T of a block pair in TMEM (pair p: p & 1)
  uint64_t* vready = dtready + 2;         // [3] V, W and the decay sums of the block ready (256 arrivals)
  uint64_t* btready = vready + 3;      // [2] B^T and C of the block in shared memory (TMA)
  uint64_t* mready = btready + 2;      // [2] M of the block in shared memory (TMA)
  uint64_t* gready = mready + 2;       // G' rescaled for the block (256 arrivals)
  uint64_t* dgready = gready + 1;      // [2] the block's state products done (G' advanced)
  uint64_t* yready = dgready + 2;      // [2] the block's Y complete
  uint64_t* yidone = yready + 2;       // Y = G' C^T done reading G' (once per block)
  uint64_t* wdone = yidone + 1;        // [3] the block's output written: V, W buffer free (256 arrivals)
  uint64_t* mma_done = wdone + 3;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* sS = reinterpret_cast<float*>(sm + OFF_S);
  volatile int* sAny = reinterpret_cast<volatile int*>(sm + OFF_ANY);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c0 = blockIdx.x * CH, b = blockIdx.y;
  const int nblk = (T - t0 + Q - 1) / Q;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NVT);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&dtready[i], 1);
      mbar_init(&btready[i], 1);
      mbar_init(&mready[i], 1);
      mbar_init(&dgready[i], 1);
      mbar_init(&yready[i], 1);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&vready[i], NVT);
      mbar_init(&wdone[i], NRT);
    }
    mbar_init(gready, NRT);
    mbar_init(yidone, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 18) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  pdl_wait();
  if (threadIdx.x == 16 * 32) {
    tma_prefetch(&tmX);
    tma_prefetch(&tmDL);
    tma_prefetch(&tmG);
    tma_prefetch(&tmWD);
  } else if (threadIdx.x == 17 * 32) {
    tma_prefetch(&tmM);
    tma_prefetch(&tmBT);
    tma_prefetch(&tmC);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(sm);

  if (warp == 16) {
    // ------------------------------------------------------------ TMA: x, gate, dt_low
    if (lane == 0) {
      int k = 0;
      for (; k < nblk; ++k) {
        const int s = k % ST;
        if (k >= ST && !mbar_wait(&empty[s], ((k / ST) - 1) & 1u, status, abort_flag)) break;
        mbar_arrive_expect_tx(&full[s], 2 * TILE_B + ka * DLC_B + (k == 0 ? ka * WDC_B : 0));
        const int t = t0 + k * Q;
        if (k == 0)
          for (int a = 0; a < ka; ++a) tma_load_2d(sm + OFF_WD + a * WDC_B, &tmWD, &full[s], a * KA, c0);
        tma_load_3d(sm + OFF_X + s * TILE_B, &tmX, &full[s], c0, t, b);
        tma_load_3d(sm + OFF_G + s * TILE_B, &tmG, &full[s], c0, t, b);
        for (int a = 0; a < ka; ++a)
          tma_load_3d(sm + OFF_DL + (a * ST + s) * DLC_B, &tmDL, &full[s], a * KA, t, b);
      }
      if (k < nblk) {  // aborted: let the copies already issued land before smem goes away
        int never = 0;
        for (int j = (k > ST ? k - ST : 0); j < k; ++j)
          mbar_wait(&full[j % ST], (j / ST) & 1u, nullptr, &never, 100000000ull);
      }
    }
  } else if (warp == 17) {
    // ------------------------------------------------------------ TMA: B^T, C, M of each
    // block (written beforehand by bc_gram_kernel) into double buffers
    if (lane == 0) {
      int nbt = 0, nm = 0;   // copies issued
      for (int k = 0; k < nblk; ++k) {
        const int i = k & 1, rec = b * nblk + k;
        // B^T / C buffer i was last read by block k - 2's state products
        if (k >= 2 && !mbar_wait(&dgready[i], ((k - 2) >> 1) & 1u, status, abort_flag)) break;
        mbar_arrive_expect_tx(&btready[i], BT_B + CC_B);
        tma_load_3d(sm + OFF_BT + i * BT_B, &tmBT, &btready[i], 0, 0, rec);
        for (int q = 0; q < 4; ++q) tma_load_3d(sm + OFF_CC + i * CC_B + q * BCC_B, &tmC, &btready[i], 32 * q, 0, rec);
        ++nbt;
        // M buffer i was last read by block k - 2's V M^T
        if (k >= 2 && !mbar_wait(&yready[i], ((k - 2) >> 1) & 1u, status, abort_flag)) break;
        mbar_arrive_expect_tx(&mready[i], MT_B);
        tma_load_3d(sm + OFF_MT + i * MT_B, &tmM, &mready[i], 0, 0, rec);
        ++nm;
      }
      // let the last copies land before shared memory goes away
      int never = 0;
      for (int j = (nbt > 2 ? nbt - 2 : 0); j < nbt; ++j)
        mbar_wait(&btready[j & 1], (j >> 1) & 1u, nullptr, &never, 100000000ull);
      for (int j = (nm > 2 ? nm - 2 : 0); j < nm; ++j)
        mbar_wait(&mready[j & 1], (j >> 1) & 1u, nullptr, &never, 100000000ull);
    }
  } else if (warp == 18) {
    // ------------------------------------------------------------ MMA issuer, in a fixed
    // order per block k (its inputs are ready, in the steady state, before it gets to them):
    //   chain(k):     Y = G' C^T, G' += V B (the state products) -> dgready
    //   pair(k + 2):  for even k, the dt projection of blocks k + 2 and k + 3 (one N = 64
    //                 product over both stages' dt_low rows) -> dtready
    //   vm(k):        Y += V M^T -> yready
    // so that while the state warps rescale G' for block k + 1 the tensor pipe works on
    // vm(k) and the dt projection, and chain(k + 1) follows as soon as G' is ready.
    // Buffer reuse: DT slots (k + 2) % 4, (k + 3) % 4 held blocks k - 2, k - 1, done with
    // by chain(k - 1) (the V/W warps read a slot before vready, the plain recurrence before
    // gready).  The V/W warps free a stage themselves once they have read its x and gate:
    // they read them only after the dt projection over its dt_low rows has completed.
    if (lane == 0) {
      // descriptors of the first stage's tiles; every other tile is a fixed offset away
      const uint64_t dDL = sdesc_sw128(sbase + OFF_DL, 16, 1024), dWD = sdesc_sw128(sbase + OFF_WD, 16, 1024),
                     dCC = sdesc_sw128(sbase + OFF_CC, 16, 1024), dBT = sdesc_sw128(sbase + OFF_BT, 16, 1024),
                     dMT = sdesc_sw128(sbase + OFF_MT, 16, 1024);
      uint32_t n_yi = 0;   // completed phases of yidone (product-form blocks only)
      // dt = W_dt dt_low^T of blocks ks, ks + 1 (ks even) into DT slots ks % 4, ks % 4 + 1:
      // the two stages' dt_low rows are adjacent (64 rows of each atom).  Without a block
      // ks + 1 the product's second half reads a stale stage into a slot nobody reads.
      auto pair = [&](int ks) -> bool {
        if (!mbar_wait(&full[ks % ST], (ks / ST) & 1u, status, abort_flag)) return false;
        if (ks + 1 < nblk && !mbar_wait(&full[(ks + 1) % ST], ((ks + 1) / ST) & 1u, status, abort_flag)) return false;
        tc_fence_after();
        const uint64_t dl = sdesc_add(dDL, (ks % ST) * DLC_B);
        const uint32_t d = tmem + COL_DT + 32 * (ks & 3);
#pragma unroll
        for (int j = 0; j < KA / 16; ++j)
          umma_bf16_ss(d, sdesc_add(dWD, 32 * j), sdesc_add(dl, 32 * j), IDESC_DT, j != 0);
        if (ka > 1) {
#pragma unroll
          for (int j = 0; j < KA / 16; ++j)
            umma_bf16_ss(d, sdesc_add(dWD, WDC_B + 32 * j), sdesc_add(dl, ST * DLC_B + 32 * j), IDESC_DT, 1u);
        }
        umma_commit(&dtready[(ks >> 1) & 1]);
        return true;
      };
      bool ok = true;
      if (nblk > 0) ok = pair(0);
      for (int k = 0; k < nblk && ok; ++k) {
        const int i = k & 1, vb = k % 3;
        // ---- chain(k)
        if (!mbar_wait(gready, k & 1u, status, abort_flag) ||
            !mbar_wait(&btready[i], (k >> 1) & 1u, status, abort_flag))
          break;
        tc_fence_after();
        const bool plain = sAny[vb] != 0;
        if (!plain) {
          const uint64_t cc = sdesc_add(dCC, i * CC_B), bt = sdesc_add(dBT, i * BT_B);
          // Y = G' C^T (K = n = 128), then G' += V B (K = s = 32, B^T rows n).  The update
          // writes the TMEM G' the first product reads as its A operand: it is issued only
          // once that product has completed (an MMA issued behind another is not held back
          // from writing TMEM the earlier one still reads)
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int j = 0; j < 4; ++j)
              umma_tf32_ts(tmem + COL_Y + 32 * i, tmem + COL_GP + 32 * q + 8 * j, sdesc_add(cc, q * BCC_B + 32 * j),
                           IDESC_Q, (q | j) != 0);
          umma_commit(yidone);
          if (!mbar_wait(yidone, n_yi & 1u, status, abort_flag)) break;
          ++n_yi;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            umma_tf32_ts(tmem + COL_GP, tmem + COL_V + 32 * vb + 8 * j, sdesc_add(bt, 32 * j), IDESC_N, 1);
        }
        umma_commit(&dgready[i]);
        // ---- the dt projection of the next pair first: the V/W warps need it as soon as
        // they are done with block k + 1, while Y(k) is wanted only after G' is rescaled
        if ((k & 1) == 0 && k + 2 < nblk && !pair(k + 2)) break;
        // ---- vm(k): Y += V M^T (K = s = 32), then Y is complete
        if (!mbar_wait(&mready[i], (k >> 1) & 1u, status, abort_flag)) break;
        tc_fence_after();
        if (!plain) {
          const uint64_t mt = sdesc_add(dMT, i * MT_B);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            umma_tf32_ts(tmem + COL_Y + 32 * i, tmem + COL_V + 32 * vb + 8 * j, sdesc_add(mt, 32 * j), IDESC_Q, 1);
        }
        umma_commit(&yready[i]);
      }
      umma_commit(mma_done);
      int never = 0;
      mbar_wait(mma_done, 0, nullptr, &never, 100000000ull);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ V/W warps: for every
    // block, dt (softplus of W_dt dt_low^T + b_dt), the half-block decay sums, and V, W
    // into TMEM buffer k % 3: V = dt x 2^(lambda - r), W = gate 2^(r - lambda) (r: lambda
    // after the first half), or for a block that runs the plain recurrence V = dt x,
    // W = gate.  Warp 8 + w: TMEM quadrant w % 4, half w / 4 of the block's steps.
    const int qd = warp & 3, half = (warp - 8) >> 2;
    const int cl = qd * 32 + lane, c = c0 + cl;
    const uint32_t tl = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    const float A2 = c < Di ? expf(a_log[c]) * 1.4426950408889634f : 0.f;  // |A| / ln 2
    const float bdt = c < Di ? b_dt[c] : 0.f;
    bool fail = false;
#pragma unroll 1
    for (int k = 0; k < nblk; ++k) {
      const int s = k % ST, vb = k % 3;
      // buffer vb was last read by the output of block k - 3 (after that block's products)
      fail = fail || !__all_sync(0xffffffffu, mbar_wait(&full[s], (k / ST) & 1u, status, abort_flag) &&
                                                  mbar_wait(&dtready[(k >> 1) & 1], (k >> 2) & 1u, status, abort_flag) &&
                                                  (k < 3 || mbar_wait(&wdone[vb], ((k - 3) / 3) & 1u, status, abort_flag)));
      // dt of this half (steps past T: dt = 0, the state stays)
      float dtv[HQ];
      if (!fail) {
        tc_fence_after();
        uint32_t z[HQ];
        tmem_ld16(tl + COL_DT + 32 * (k & 3) + HQ * half, z);
        tmem_wait_ld();
        const int t_end = T - (t0 + k * Q + HQ * half);
#pragma unroll
        for (int j = 0; j < HQ; j += 2) {
          float2 d = softplus2(make_float2(__uint_as_float(z[j]) + bdt, __uint_as_float(z[j + 1]) + bdt));
          if (j >= t_end) d.x = 0.f;
          if (j + 1 >= t_end) d.y = 0.f;
          dtv[j] = d.x;
          dtv[j + 1] = d.y;
        }
      } else {
#pragma unroll
        for (int j = 0; j < HQ; ++j) dtv[j] = 0.f;
      }
      float2 S2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int j = 0; j < HQ; j += 2) S2 = __ffma2_rn(make_float2(A2, A2), make_float2(dtv[j], dtv[j + 1]), S2);
      const float S = S2.x + S2.y;
      float* ss = sS + (k & 1) * 2 * CH;
      ss[half * CH + cl] = S;
      // one reduction in the common case: "some channel needs the plain recurrence or some
      // thread failed"; only when it is set, a second one tells the two apart (both
      // uniform over the V/W threads, which therefore leave the loop together)
      const bool any = bar_red_or(1, NVT, fail || !(S <= kRange));
      const bool stop = any && bar_red_or(1, NVT, fail);
      const float S0 = ss[cl];
      if (!fail) {
        // x and gate of this half (shared loads issued first), the running decay
        // mu = lambda - r (one dependent FMA per step), then the exponentials, which are
        // independent of one another; the block-uniform branch stays outside the loops
        const uint32_t xa = sbase + OFF_X + s * TILE_B + cl * 2 + HQ * half * 256;
        const uint32_t ga = sbase + OFF_G + s * TILE_B + cl * 2 + HQ * half * 256;
        float xv[HQ], gv[HQ];
#pragma unroll
        for (int j = 0; j < HQ; ++j) {
          xv[j] = bf2f(static_cast<uint16_t>(lds_u16(xa + j * 256)));
          gv[j] = bf2f(static_cast<uint16_t>(lds_u16(ga + j * 256)));
        }
        mbar_arrive(&empty[s]);   // x and gate are in registers: the stage can be refilled
        uint32_t vr[HQ], wr[HQ];
        if (!any) {
          float mu[HQ];
          float m = half ? 0.f : -S0;
#pragma unroll
          for (int j = 0; j < HQ; ++j) {
            m = fmaf(A2, dtv[j], m);
            mu[j] = m;
          }
#pragma unroll
          for (int j = 0; j < HQ; j += 2) {
            const float2 u = __fmul2_rn(make_float2(dtv[j], dtv[j + 1]), make_float2(xv[j], xv[j + 1]));
            const float2 v = __fmul2_rn(u, make_float2(ex2_approx(mu[j]), ex2_approx(mu[j + 1])));
            const float2 w =
                __fmul2_rn(make_float2(gv[j], gv[j + 1]), make_float2(ex2_approx(-mu[j]), ex2_approx(-mu[j + 1])));
            vr[j] = tf32_round(v.x);
            vr[j + 1] = tf32_round(v.y);
            wr[j] = __float_as_uint(w.x);
            wr[j + 1] = __float_as_uint(w.y);
          }
        } else {
#pragma unroll
          for (int j = 0; j < HQ; ++j) {
            vr[j] = __float_as_uint(dtv[j] * xv[j]);
            wr[j] = __float_as_uint(gv[j]);
          }
        }
        tmem_st16(tl + COL_V + 32 * vb + HQ * half, vr);
        tmem_st16(tl + COL_W + 32 * vb + HQ * half, wr);
        tmem_wait_st();
      }
      if (fail) mbar_arrive(&empty[s]);   // (skipped above)
      if (warp == 8 && lane == 0) sAny[vb] = any ? 1 : 0;
      tc_fence_before();
      mbar_arrive(&vready[vb]);
      if (stop) break;
    }
  } else {
    // ------------------------------------------------------------ state warps: per block,
    // rescale G' (or run the plain recurrence), hand the block to the MMA thread, then
    // write the previous block's y.  Warp w: TMEM quadrant w % 4, half w / 4 of G''s
    // columns and of the block's output rows.
    const int qd = warp & 3, half = warp >> 2;
    const int cl = qd * 32 + lane, c = c0 + cl;
    const uint32_t tl = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    const float A2 = c < Di ? expf(a_log[c]) * 1.4426950408889634f : 0.f;  // |A| / ln 2
    const float bdt = c < Di ? b_dt[c] : 0.f;
    __nv_bfloat16* ycol = y + static_cast<long long>(b) * T * y_ld + c;
    __nv_bfloat16* ybase = y + static_cast<long long>(b) * T * y_ld;
    const int c4 = c0 + qd * 32 + (lane & ~3);   // this lane's 4-channel store group
    bool fail = false;
    // the state entering row t0, columns [64 half, 64 half + 64) (raw: the first block
    // applies only its own scale)
#pragma unroll 1
    for (int part = 0; part < 2; ++part) {
      const int n0 = 64 * half + 32 * part;
      uint32_t hz[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) hz[j] = 0u;
      if (h0 && c < Di) {
        const float4* hp = reinterpret_cast<const float4*>(h0 + b * h0_bstride + static_cast<long long>(c) * NS + n0);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 v = hp[j];
          hz[4 * j] = __float_as_uint(v.x);
          hz[4 * j + 1] = __float_as_uint(v.y);
          hz[4 * j + 2] = __float_as_uint(v.z);
          hz[4 * j + 3] = __float_as_uint(v.w);
        }
      }
      tmem_st32(tl + COL_GP + n0, hz);
    }
    tmem_wait_st();
    tc_fence_before();
    // y = W * Y over this half's 16 rows of block jb
    auto out_block = [&](int jb) {
      const int i = jb & 1;
      tc_fence_after();
      uint32_t yv[HQ], wv[HQ];
      tmem_ld16(tl + COL_Y + 32 * i + HQ * half, yv);
      tmem_ld16(tl + COL_W + 32 * (jb % 3) + HQ * half, wv);
      tmem_wait_ld();
      float o[HQ];
#pragma unroll
      for (int j = 0; j < HQ; ++j) o[j] = __uint_as_float(yv[j]) * __uint_as_float(wv[j]);
      store_y16(ybase, y_ld, t0 + jb * Q + HQ * half, T, c4, c4 < Di, o);
    };

    float pS1 = 0.f;        // the previous block's second-half decay sum
    bool prev_any = true;   // the previous block left the raw state in G' (so does the start)
#pragma unroll 1
    for (int k = 0; k < nblk; ++k) {
      // ---- block k's sums and flag (V/W done) and G' (block k - 1's products done)
      if (k > 0)
        fail = fail || !__all_sync(0xffffffffu, mbar_wait(&dgready[(k - 1) & 1], ((k - 1) >> 1) & 1u, status, abort_flag));
      fail = fail || !__all_sync(0xffffffffu, mbar_wait(&vready[k % 3], (k / 3) & 1u, status, abort_flag));
      if (fail) break;
      const float* ss = sS + (k & 1) * 2 * CH;
      const float cS0 = ss[cl], cS1 = ss[CH + cl];
      const bool c_any = sAny[k % 3] != 0;
      tc_fence_after();
      if (!c_any) {
        // G' <- 2^-e_in 2^-e_out G'; one multiply while 2^-(e_in + e_out) is a normal float
        const float e_in = prev_any ? 0.f : pS1, e_out = cS0;
        const bool one = __all_sync(0xffffffffu, e_in + e_out < 120.f);
        const float f1 = ex2_approx(one ? -(e_in + e_out) : -e_in), f2 = one ? 1.f : ex2_approx(-e_out);
        const float2 fa = make_float2(f1, f1), fb = make_float2(f2, f2);
        // both 32-column pieces in flight at once: one load wait, one store wait
        const uint32_t col = tl + COL_GP + 64 * half;
        uint32_t g[64];
        tmem_ld32(col, *reinterpret_cast<uint32_t(*)[32]>(&g[0]));
        tmem_ld32(col + 32, *reinterpret_cast<uint32_t(*)[32]>(&g[32]));
        tmem_wait_ld();
        if (one) {
#pragma unroll
          for (int j = 0; j < 64; j += 2) {
            const float2 v = __fmul2_rn(make_float2(__uint_as_float(g[j]), __uint_as_float(g[j + 1])), fa);
            g[j] = __float_as_uint(v.x);
            g[j + 1] = __float_as_uint(v.y);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 64; j += 2) {
            const float2 v =
                __fmul2_rn(__fmul2_rn(make_float2(__uint_as_float(g[j]), __uint_as_float(g[j + 1])), fa), fb);
            g[j] = __float_as_uint(v.x);
            g[j + 1] = __float_as_uint(v.y);
          }
        }
        tmem_st32(col, *reinterpret_cast<uint32_t(*)[32]>(&g[0]));
        tmem_st32(col + 32, *reinterpret_cast<uint32_t(*)[32]>(&g[32]));
        tmem_wait_st();
      } else if (half == 1) {
        // ---- large decays: the plain recurrence over block k by the half-1 warps (one
        // thread per channel, all 128 state columns, 8 at a time).  G' holds 2^S1 times
        // the state after a product-form block: that factor is taken out as it is loaded.
        const float f_in = prev_any ? 1.f : ex2_approx(-pS1);
        const int i = k & 1, vb = k % 3;
        fail = !__all_sync(0xffffffffu, mbar_wait(&btready[i], (k >> 1) & 1u, status, abort_flag));
        if (!fail) {
          tc_fence_after();
          const uint8_t* bt = sm + OFF_BT + i * BT_B;
          const uint8_t* cc = sm + OFF_CC + i * CC_B;
#pragma unroll 1
          for (int th = 0; th < Q; th += QQ) {
            uint32_t zq[QQ], uq[QQ], gq[QQ];
            tmem_ld8(tl + COL_DT + 32 * (k & 3) + th, zq);
            tmem_ld8(tl + COL_V + 32 * vb + th, uq);
            tmem_ld8(tl + COL_W + 32 * vb + th, gq);
            tmem_wait_ld();
            const int t_end = T - (t0 + k * Q + th);
            float a[QQ], yq[QQ];
#pragma unroll
            for (int j = 0; j < QQ; ++j) {
              const float dt = j < t_end ? softplus_f(__uint_as_float(zq[j]) + bdt) : 0.f;
              a[j] = ex2_approx(-A2 * dt);
              yq[j] = 0.f;
            }
            const float fq = th == 0 ? f_in : 1.f;
#pragma unroll 1
            for (int q = 0; q < NS / 8; ++q) {
              uint32_t hr[8];
              tmem_ld8(tl + COL_GP + 8 * q, hr);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 8; ++j) hr[j] = __float_as_uint(__uint_as_float(hr[j]) * fq);
#pragma unroll
              for (int tt = 0; tt < QQ; ++tt) {
                const int t = th + tt;
                const float u = __uint_as_float(uq[tt]);
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < 8; j += 4) {
                  const float4 cv = *reinterpret_cast<const float4*>(cc + cc_off(t, 8 * q + j));
                  const float cq[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    const float bn = *reinterpret_cast<const float*>(bt + bt_off(8 * q + j + e, t));
                    const float h = fmaf(a[tt], __uint_as_float(hr[j + e]), u * bn);
                    hr[j + e] = __float_as_uint(h);
                    acc = fmaf(cq[e], h, acc);
                  }
                }
                yq[tt] += acc;
              }
              tmem_st8(tl + COL_GP + 8 * q, hr);
              tmem_wait_st();
            }
            if (c < Di) {
#pragma unroll
              for (int j = 0; j < QQ; ++j) {
                const int t = t0 + k * Q + th + j;
                if (t < T) ycol[static_cast<long long>(t) * y_ld] = __float2bfloat16_rn(__uint_as_float(gq[j]) * yq[j]);
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(gready);
      if (fail) break;
      // ---- output of block k - 1.  Every phase of yready is waited for, even after a
      // plain block (whose y went out already): a skipped phase would let the parity test
      // of the next wait on the same barrier pass a phase early
      if (k > 0) {
        const int jb = k - 1;
        fail = !__all_sync(0xffffffffu, mbar_wait(&yready[jb & 1], (jb >> 1) & 1u, status, abort_flag));
        if (fail) break;
        if (!prev_any) out_block(jb);
        mbar_arrive(&wdone[jb % 3]);   // W and V of block k - 1 are free
      }
      pS1 = cS1;
      prev_any = c_any;
    }
    // ---- output of the last block and the state after the last row
    if (__all_sync(0xffffffffu, !fail && nblk > 0 && !*abort_flag)) {
      const int jb = nblk - 1, i = jb & 1;
      const bool got = __all_sync(0xffffffffu, mbar_wait(&dgready[i], (jb >> 1) & 1u, status, abort_flag));
      if (got && !prev_any && __all_sync(0xffffffffu, mbar_wait(&yready[i], (jb >> 1) & 1u, status, abort_flag)))
        out_block(jb);
      if (got && h_out) {
        // 2^-S1 (G' + dG) after a product-form block, the raw state after a plain one
        const float f = prev_any ? 1.f : ex2_approx(-pS1);
        tc_fence_after();
#pragma unroll 1
        for (int part = 0; part < 2; ++part) {
          const int n0 = 64 * half + 32 * part;
          uint32_t g[32];
          tmem_ld32(tl + COL_GP + n0, g);
          tmem_wait_ld();
          if (c < Di) {
            float4* ho = reinterpret_cast<float4*>(h_out + (static_cast<long long>(b) * Di + c) * NS + n0);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              ho[j] = make_float4(__uint_as_float(g[4 * j]) * f, __uint_as_float(g[4 * j + 1]) * f,
                                  __uint_as_float(g[4 * j + 2]) * f, __uint_as_float(g[4 * j + 3]) * f);
          }
        }
      }
    } else if (nblk == 0 && h_out && c < Di && h0) {
      // no rows to scan: the state passes through
      const float* hp = h0 + b * h0_bstride + static_cast<long long>(c) * NS + 64 * half;
      float* ho = h_out + (static_cast<long long>(b) * Di + c) * NS + 64 * half;
      for (int j = 0; j < 64; ++j) ho[j] = hp[j];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 18) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

cudaError_t launch_tc128(const ScanDesc& s, cudaStream_t st) {
  if (!s.mgram || !a16(s.mgram)) return cudaErrorInvalidValue;
  const int nblk = (s.T - s.t0 + Q - 1) / Q;
  const long long nrec = static_cast<long long>(s.batch) * (nblk > 0 ? nblk : 1);
  uint8_t* rec = static_cast<uint8_t*>(s.mgram);
  CUtensorMap tx, td, tg, tw, tm, tbt, tc;
  const bool ok =
      map_rec_f32(&tm, rec, Q, Q, Q * 4, nrec, GREC_B, Q, Q) &&
      map_rec_f32(&tbt, rec + MT_B, Q, NS, Q * 4, nrec, GREC_B, Q, NS) &&
      map_rec_f32(&tc, rec + MT_B + BT_B, NS, Q, NS * 4, nrec, GREC_B, 32, Q) &&
      map3d(&tx, s.x, false, s.batch, s.T, s.d_inner, s.d_inner, CH, Q, CU_TENSOR_MAP_SWIZZLE_NONE) &&
      map3d(&tg, s.gate, false, s.batch, s.T, s.d_inner, s.d_inner, CH, Q, CU_TENSOR_MAP_SWIZZLE_NONE) &&
      map3d(&td, s.dt_low, false, s.batch, s.T, s.dt_rank, s.dt_rank, KA, Q, CU_TENSOR_MAP_SWIZZLE_128B) &&
      map2d_sw128(&tw, s.w_dt, s.d_inner, s.dt_rank, s.dt_rank, KA, CH);
  if (!ok) return cudaErrorNotSupported;
  static std::atomic<uint64_t> attr_done{0};
  if (cudaError_t e = smem_attr_once(scan_tc128_kernel, SMEM_TOTAL, attr_done)) return e;
  const int ka = (s.dt_rank + KA - 1) / KA;
  if (nblk > 0) {
    if (cudaError_t e = launch(bc_gram_kernel, dim3(nblk, s.batch), dim3(256), 0, st, s.bc, s.T, s.t0, nblk, rec))
      return e;
  }
  dim3 grid((s.d_inner + CH - 1) / CH, s.batch);
  return launch(scan_tc128_kernel, grid, dim3(NTHR2), SMEM_TOTAL, st, tx, td, tg, tw, tm, tbt, tc, s.a_log, s.b_dt,
                static_cast<__nv_bfloat16*>(s.y), s.y_ld, s.T, s.d_inner, ka, s.h_out, s.t0, s.h0, s.h0_bstride,
                s.status);
}
}  // namespace t128

}  // namespace

bool scan_tc_fuses_dt(const ScanDesc& s) {
  const bool rank_ok = s.d_state == NST ? s.dt_rank == KR
                                        : (s.d_state == t128::NS && s.dt_rank >= 8 && s.dt_rank <= 2 * t128::KA &&
                                           s.dt_rank % 8 == 0);
  return s.bf16 && rank_ok && !s.a_per_state && (s.d_inner * 2) % 16 == 0 && (s.y_ld * 2) % 16 == 0 && a16(s.x) &&
         a16(s.gate) && a16(s.bc) && a16(s.y) && a16(s.dt_low) && a16(s.w_dt) && s.b_dt != nullptr &&
         (s.h0 == nullptr || a16(s.h0)) && (s.h_out == nullptr || a16(s.h_out));
}

size_t scan_mgram_bytes(const ScanDesc& s) {
  if (s.d_state != t128::NS || !s.dt_low || s.T <= s.t0) return 0;
  const size_t nblk = static_cast<size_t>(s.T - s.t0 + t128::Q - 1) / t128::Q;
  return static_cast<size_t>(s.batch) * nblk * t128::GREC_B;
}

// bf16, d_state 16 or 128, 16-byte aligned operands and row strides (checked by the
// caller; with dt_low set, scan_tc_fuses_dt).  d_state 128 runs only with the dt
// projection fused.  cudaErrorNotSupported when the configuration is not these kernels'.
cudaError_t launch_scan_tc(const ScanDesc& s, cudaStream_t st) {
  if (!s.bf16 || s.a_per_state) return cudaErrorNotSupported;
  if (s.d_state == t128::NS)
    return s.dt_low && scan_tc_fuses_dt(s) ? t128::launch_tc128(s, st) : cudaErrorNotSupported;
  if (s.d_state != NST) return cudaErrorNotSupported;
  if (s.dt_low) return scan_tc_fuses_dt(s) ? launch_tc<true>(s, st) : cudaErrorNotSupported;
  return launch_tc<false>(s, st);
}

}  // namespace hy
