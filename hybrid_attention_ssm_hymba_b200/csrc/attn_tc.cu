// attn_tc.cu -- attention heads of the hybrid-head layer on the sm_100a tensor cores
// (blog.outta.ai Hymba review, "Design formulation": Y_attn = softmax(Q K^T) V;
// "Combine global and local attention": sliding-window attention in most layers;
// "Meta Tokens": the meta tokens stay visible to every query).  A query i of a
// sequence sees key j iff j <= i and (window < 0 or i - j <= window or j < n_meta);
// query head h reads K/V head h / (Hq / Hkv) (GQA).  Scale 1/sqrt(head_dim).
//
// One CTA per (128-query tile, query head, sequence); 192 threads:
//   warp 0      TMA producer: Q once, then K_j and V_j into two 2-deep rings
//   warp 1      TMEM allocator + UMMA issuer: S_j = Q K_j^T into one of two TMEM
//               S buffers (issued two blocks ahead), O_j = P_j V_j into TMEM
//   warps 2..5  softmax: one query row per thread; S_j read from TMEM once; fp32 row
//               max and sum; P_j in bf16 into one of two swizzled smem tiles (the A
//               operand of P V); O accumulates in TMEM across blocks, rescaled in place
//               only when the running max grows by more than 2^8; final O / l as bf16.
// K/V blocks with no visible pair are never loaded: the block list is the meta
// blocks plus the window blocks.  Only blocks that straddle the mask boundary pay
// for the elementwise mask.
#include "hy_common.cuh"
#include "hy_kernels.h"

namespace hy {
namespace {

constexpr int BQ = 128, BKV = 128, DH = 128;
constexpr int TILE_BYTES = 128 * DH * 2;  // 32 KB: a [128 x 128] bf16 tile = 2 swizzled 64-column halves
constexpr int HALF = 128 * 64 * 2;        // 16 KB
constexpr int SMEM_BYTES = 7 * TILE_BYTES + 1024 + 256;
constexpr uint32_t IDESC_QK = idesc_bf16(BQ, BKV, false, false);  // A=Q (K-major), B=K (K-major)
constexpr uint32_t IDESC_PV = idesc_bf16(BQ, DH, false, true);    // A=P (K-major), B=V (MN-major)

struct AttnParams {
  int T, Hq, Hkv, n_meta, window;
  int q_tiles;
  __nv_bfloat16* out;
  long long out_ld;
  float scale_log2;  // log2(e) / sqrt(dh)
  unsigned* status;
};

struct BlockList {
  int first, wlo, n;  // blocks [0, first) then [wlo, wlo + n - first)
  __device__ __forceinline__ int block(int idx) const { return idx < first ? idx : wlo + (idx - first); }
};

__device__ __forceinline__ BlockList make_blocks(const AttnParams& p, int q0) {
  BlockList bl;
  const int last_row = min(q0 + BQ - 1, p.T - 1);
  const int hi = last_row / BKV;
  if (p.window < 0) {
    bl.first = 0;
    bl.wlo = 0;
  } else {
    const int mb = (p.n_meta + BKV - 1) / BKV;
    bl.wlo = max(0, q0 - p.window) / BKV;
    bl.first = min(mb, bl.wlo);
  }
  bl.n = bl.first + (hi - bl.wlo + 1);
  return bl;
}

__device__ __forceinline__ bool visible(int i, int j, int n_meta, int window) {
  return j <= i && (window < 0 || i - j <= window || j < n_meta);
}

// Three-input fp32 maximum (sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// Maximum of a 64-value half row (fp32 bit patterns): eight independent chains of
// three-input maxima, so the reduction is 5 dependent steps deep instead of 64.
__device__ __forceinline__ float row_max64(const uint32_t (&sv)[64]) {
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = fmaxf(__uint_as_float(sv[i]), __uint_as_float(sv[i + 8]));
#pragma unroll
  for (int e = 16; e < 64; e += 16)
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = max3f(m[i], __uint_as_float(sv[e + i]), __uint_as_float(sv[e + 8 + i]));
  return max3f(max3f(m[0], m[1], m[2]), max3f(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}
// P = 2^(S scale - m_ref) for a 64-value half row, packed in place as bf16 pairs
// (sv[q] <- (p[2q], p[2q+1]); reads index >= q first); returns the sum of the fp32
// values.  Paired scale-and-subtract, four independent partial sums.
__device__ __forceinline__ float row_exp64(uint32_t (&sv)[64], float scale_log2, float m_ref) {
  const float2 sc = make_float2(scale_log2, scale_log2), nm = make_float2(-m_ref, -m_ref);
  float2 acc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.f, 0.f);
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[2 * q]), __uint_as_float(sv[2 * q + 1])), sc, nm);
    const float2 pq = make_float2(ex2_approx(x.x), ex2_approx(x.y));
    acc[q & 3] = __fadd2_rn(acc[q & 3], pq);
    sv[q] = pack_bf16(pq.x, pq.y);
  }
  const float2 t = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
  return t.x + t.y;
}

__global__ void __launch_bounds__(192, 1)
    attn_fwd_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* sQ = smem_raw + pad;
  uint8_t* sK = sQ + TILE_BYTES;      // 2 stages
  uint8_t* sV = sK + 2 * TILE_BYTES;  // 2 stages
  uint8_t* sP = sV + 2 * TILE_BYTES;  // 2 buffers
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + 2 * TILE_BYTES);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;   // [2]
  uint64_t* k_empty = bars + 3;  // [2]
  uint64_t* v_full = bars + 5;   // [2]
  uint64_t* v_empty = bars + 7;  // [2]
  uint64_t* s_full = bars + 9;   // [2]
  uint64_t* s_free = bars + 11;  // [2]
  uint64_t* p_full = bars + 13;  // [2]
  uint64_t* p_free = bars + 15;  // [2]
  uint64_t* o_done = bars + 17;  // completes once per P V
  uint64_t* mma_done = bars + 18;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 19);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = p.q_tiles - 1 - static_cast<int>(blockIdx.x);  // longest tiles first
  const int h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (p.Hq / p.Hkv);
  const int q0 = qt * BQ;
  const BlockList bl = make_blocks(p, q0);
  const int n = bl.n;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 128);
      mbar_init(&p_full[s], 128);
      mbar_init(&p_free[s], 1);
    }
    mbar_init(o_done, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch(&tmQ);
    tma_prefetch(&tmK);
    tma_prefetch(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tS = tmem_base, tO = tmem_base + 256;  // S: 2 x 128 columns, O: 128 columns

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      uint32_t k_iss = 0, v_iss = 0, k_par = 0, v_par = 0;
      bool ok = true;
      mbar_arrive_expect_tx(q_full, TILE_BYTES);
      tma_load_3d(sQ, &tmQ, q_full, h * DH, q0, b);
      tma_load_3d(sQ + HALF, &tmQ, q_full, h * DH + 64, q0, b);
      auto issue_kv = [&](uint8_t* ring, const CUtensorMap* map, uint64_t* full, uint64_t* empty, int j,
                          uint32_t& iss, uint32_t& par) -> bool {
        const int s = j & 1;
        if (!mbar_wait(&empty[s], ((j >> 1) & 1) ^ 1u, p.status, abort_flag)) return false;
        mbar_arrive_expect_tx(&full[s], TILE_BYTES);
        const int k0 = bl.block(j) * BKV;
        tma_load_3d(ring + s * TILE_BYTES, map, &full[s], kvh * DH, k0, b);
        tma_load_3d(ring + s * TILE_BYTES + HALF, map, &full[s], kvh * DH + 64, k0, b);
        iss |= 1u << s;
        par = (par & ~(1u << s)) | (static_cast<uint32_t>((j >> 1) & 1) << s);
        return true;
      };
      // consumption order of the UMMA issuer: K0 K1 V0 K2 V1 K3 V2 ...
      int kj = 0, vj = 0;
      while (ok && kj < n && kj < 2) ok = issue_kv(sK, &tmK, k_full, k_empty, kj++, k_iss, k_par);
      while (ok && vj < n) {
        ok = issue_kv(sV, &tmV, v_full, v_empty, vj++, v_iss, v_par);
        if (ok && kj < n) ok = issue_kv(sK, &tmK, k_full, k_empty, kj++, k_iss, k_par);
      }
      int never = 0;
      // drain: every issued copy lands before the CTA may exit
      for (int s = 0; s < 2; ++s) {
        if (k_iss & (1u << s)) mbar_wait(&k_full[s], (k_par >> s) & 1u, nullptr, &never, 100000000ull);
        if (v_iss & (1u << s)) mbar_wait(&v_full[s], (v_par >> s) & 1u, nullptr, &never, 100000000ull);
      }
      mbar_wait(q_full, 0, nullptr, &never, 100000000ull);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- UMMA issuer
      bool ok = mbar_wait(q_full, 0, p.status, abort_flag);
      // descriptors of the Q tile and the first K, P and V tiles; the rest are fixed offsets
      const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024), dK = sdesc_sw128(smem_u32(sK), 16, 1024),
                     dP = sdesc_sw128(smem_u32(sP), 16, 1024), dV = sdesc_sw128(smem_u32(sV), HALF, 1024);
      auto issue_s = [&](int j) -> bool {
        const int s = j & 1;
        const uint32_t par = (j >> 1) & 1;
        if (!mbar_wait(&k_full[s], par, p.status, abort_flag)) return false;
        if (!mbar_wait(&s_free[s], par ^ 1u, p.status, abort_flag)) return false;
        tc_fence_after();
        const uint64_t kd = sdesc_add(dK, s * TILE_BYTES);
#pragma unroll
        for (int k = 0; k < DH / 16; ++k) {
          const uint32_t off = (k >> 2) * HALF + (k & 3) * 32;
          umma_bf16_ss(tS + s * 128, sdesc_add(dQ, off), sdesc_add(kd, off), IDESC_QK, k != 0 ? 1u : 0u);
        }
        umma_commit(&s_full[s]);
        umma_commit(&k_empty[s]);
        return true;
      };
      if (ok && n > 0) ok = issue_s(0);
      if (ok && n > 1) ok = issue_s(1);
      for (int j = 0; ok && j < n; ++j) {
        const int s = j & 1;
        const uint32_t par = (j >> 1) & 1;
        if (!mbar_wait(&p_full[s], par, p.status, abort_flag)) break;
        if (!mbar_wait(&v_full[s], par, p.status, abort_flag)) break;
        tc_fence_after();
        const uint64_t pd = sdesc_add(dP, s * TILE_BYTES), vd = sdesc_add(dV, s * TILE_BYTES);
#pragma unroll
        for (int k = 0; k < BKV / 16; ++k) {
          const uint32_t a_off = (k >> 2) * HALF + (k & 3) * 32;  // P: K-major, keys 16k..16k+15
          const uint32_t b_off = k * 16 * 128;                      // V: MN-major, key rows 16k..
          umma_bf16_ss(tO, sdesc_add(pd, a_off), sdesc_add(vd, b_off), IDESC_PV, (j | k) != 0 ? 1u : 0u);
        }
        umma_commit(o_done);
        umma_commit(&p_free[s]);
        umma_commit(&v_empty[s]);
        if (j + 2 < n) ok = issue_s(j + 2);
      }
      umma_commit(mma_done);
      int never = 0;
      mbar_wait(mma_done, 0, nullptr, &never, 100000000ull);
    }
  } else {
    // ------------------------------------------------------------------ softmax
    // One query row per thread.  O accumulates in TMEM across KV blocks with a lazy
    // rescale: P is taken relative to the running max m_used, which moves (and O, l
    // are rescaled by exp2(m_old - m_new)) only when a block raises the row max by
    // more than 2^8, so P stays below 256 and the rescale is rare.
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int i = q0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    constexpr float kRescaleLog2 = 8.0f;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int s = j & 1;
      const uint32_t par = (j >> 1) & 1;
      const int k0 = bl.block(j) * BKV;
      const bool need_mask =
          !((k0 + BKV - 1 <= q0) && (p.window < 0 || q0 + BQ - 1 - k0 <= p.window || k0 + BKV - 1 < p.n_meta));
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[s], par, p.status, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sv[128];
      {
        uint32_t (&c0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[0]);
        uint32_t (&c1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[32]);
        uint32_t (&c2)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[64]);
        uint32_t (&c3)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[96]);
        const uint32_t sb = tS + s * 128 + lane_off;
        tmem_ld32(sb, c0);
        tmem_ld32(sb + 32, c1);
        tmem_ld32(sb + 64, c2);
        tmem_ld32(sb + 96, c3);
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(&s_free[s]);
      if (need_mask) {
#pragma unroll
        for (int e = 0; e < 128; ++e)
          if (!visible(i, k0 + e, p.n_meta, p.window)) sv[e] = __float_as_uint(-INFINITY);
      }
      float mx = -INFINITY;
#pragma unroll
      for (int e = 0; e < 128; ++e) mx = fmaxf(mx, __uint_as_float(sv[e]));
      const float m_cand = mx * p.scale_log2;
      const bool need = m_cand > m_used + kRescaleLog2;
      float alpha = 1.f;
      if (need) {
        alpha = ex2_approx(m_used - m_cand);  // 0 when m_used is -inf
        m_used = m_cand;
      }
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // rescale the O rows accumulated so far (all earlier P V must have landed)
        if (!__all_sync(0xffffffffu, mbar_wait(o_done, (j - 1) & 1, p.status, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tO + lane_off + c * 32, o);
        }
        tmem_wait_st();
      }
      const float m_ref = (m_used == -INFINITY) ? 0.f : m_used;
      float sum = 0.f;
      if (!__all_sync(0xffffffffu, mbar_wait(&p_free[s], par ^ 1u, p.status, abort_flag))) {
        ok = false;
        break;
      }
      uint8_t* prow = sP + s * TILE_BYTES + r * 128;
#pragma unroll
      for (int chunk = 0; chunk < 16; ++chunk) {  // 16-byte chunk = keys 8*chunk .. 8*chunk+7
        uint32_t pk[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(sv[8 * chunk + 2 * q]), p.scale_log2, -m_ref));
          const float p1 = ex2_approx(fmaf(__uint_as_float(sv[8 * chunk + 2 * q + 1]), p.scale_log2, -m_ref));
          sum += p0 + p1;
          pk[q] = pack_bf16(p0, p1);
        }
        uint8_t* dst = prow + (chunk >> 3) * HALF + (((chunk & 7) ^ (r & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      l = fmaf(l, alpha, sum);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[s]);
    }
    if (ok && n > 0 && __all_sync(0xffffffffu, mbar_wait(o_done, (n - 1) & 1, p.status, abort_flag))) {
      tc_fence_after();
      const float inv = 1.f / l;
      __nv_bfloat16* orow = p.out + (static_cast<long long>(b) * p.T + i) * p.out_ld + h * DH;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + lane_off + c * 32, o);
        tmem_wait_ld();
        if (i < p.T) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pack_bf16(__uint_as_float(o[8 * q]) * inv, __uint_as_float(o[8 * q + 1]) * inv),
                                pack_bf16(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv),
                                pack_bf16(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv),
                                pack_bf16(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ---------------------------------------------------------------------------------
// Two query heads of one KV head per CTA (GQA groups of even size): the two softmax
// groups ping-pong against the tensor core and share every K/V tile.
//   warp 0      TMA producer: Q of both heads once, then K_j / V_j (2-deep rings)
//   warp 1      UMMA issuer, per block j: P_a V_j, S_a(j+1), P_b V_j, S_b(j+1)
//   warps 2..9  softmax of head a, warps 10..17 softmax of head b: two threads per query
//               row (warps w and w + 4 share a TMEM lane quadrant), each over 64 of the
//               block's 128 keys and 64 of O's columns; the row maximum is exchanged
//               through shared memory once per block, the row sum once at the end
// TMEM (512 columns): S_a | S_b | O_a | O_b, 128 fp32 columns each.  P_x(j) (bf16,
// two keys per 32-bit column) is written over the consumed S_x(j) columns and read
// by the P V instruction straight from TMEM, so P never touches shared memory; S_x(j+1)
// is issued only after P_x V_j has completed.  O accumulates in TMEM with the same
// lazy rescale as the one-head kernel.
constexpr int SMEM2_BYTES = 6 * TILE_BYTES + 1024 + 256 + 2 * 2 * 2 * 128 * 4 + 2 * 2 * 128 * 4;

__global__ void __launch_bounds__(576, 1)
    attn_fwd_tc2(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* sQ = smem_raw + pad;       // 2 heads
  uint8_t* sK = sQ + 2 * TILE_BYTES;  // 2 stages
  uint8_t* sV = sK + 2 * TILE_BYTES;  // 2 stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + 2 * TILE_BYTES);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;   // [2]
  uint64_t* k_empty = bars + 3;  // [2]
  uint64_t* v_full = bars + 5;   // [2]
  uint64_t* v_empty = bars + 7;  // [2]
  uint64_t* s_full = bars + 9;   // [head]
  uint64_t* p_full = bars + 11;  // [head]
  uint64_t* o_done = bars + 13;  // [head], completes once per P V
  uint64_t* mma_done = bars + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* smax = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 256);  // [2 j][2 head][2 half][128 row]
  float* slsum = smax + 2 * 2 * 2 * 128;                                           // [2 head][2 half][128 row]

  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = p.q_tiles - 1 - static_cast<int>(blockIdx.x);  // longest tiles first
  const int h0 = 2 * blockIdx.y, b = blockIdx.z;                // heads h0, h0 + 1
  const int kvh = h0 / (p.Hq / p.Hkv);
  const int q0 = qt * BQ;
  const BlockList bl = make_blocks(p, q0);
  const int n = bl.n;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 256);
      mbar_init(&o_done[s], 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch(&tmQ);
    tma_prefetch(&tmK);
    tma_prefetch(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      uint32_t k_iss = 0, v_iss = 0, k_par = 0, v_par = 0;
      bool ok = true;
      mbar_arrive_expect_tx(q_full, 2 * TILE_BYTES);
      for (int x = 0; x < 2; ++x) {
        tma_load_3d(sQ + x * TILE_BYTES, &tmQ, q_full, (h0 + x) * DH, q0, b);
        tma_load_3d(sQ + x * TILE_BYTES + HALF, &tmQ, q_full, (h0 + x) * DH + 64, q0, b);
      }
      auto issue_kv = [&](uint8_t* ring, const CUtensorMap* map, uint64_t* full, uint64_t* empty, int j,
                          uint32_t& iss, uint32_t& par) -> bool {
        const int s = j & 1;
        if (!mbar_wait(&empty[s], ((j >> 1) & 1) ^ 1u, p.status, abort_flag)) return false;
        mbar_arrive_expect_tx(&full[s], TILE_BYTES);
        const int k0 = bl.block(j) * BKV;
        tma_load_3d(ring + s * TILE_BYTES, map, &full[s], kvh * DH, k0, b);
        tma_load_3d(ring + s * TILE_BYTES + HALF, map, &full[s], kvh * DH + 64, k0, b);
        iss |= 1u << s;
        par = (par & ~(1u << s)) | (static_cast<uint32_t>((j >> 1) & 1) << s);
        return true;
      };
      // first-use order of the UMMA issuer: K0 V0 K1 V1 K2 V2 ...
      for (int j = 0; ok && j < n; ++j) {
        ok = issue_kv(sK, &tmK, k_full, k_empty, j, k_iss, k_par);
        if (ok) ok = issue_kv(sV, &tmV, v_full, v_empty, j, v_iss, v_par);
      }
      int never = 0;
      for (int s = 0; s < 2; ++s) {
        if (k_iss & (1u << s)) mbar_wait(&k_full[s], (k_par >> s) & 1u, nullptr, &never, 100000000ull);
        if (v_iss & (1u << s)) mbar_wait(&v_full[s], (v_par >> s) & 1u, nullptr, &never, 100000000ull);
      }
      mbar_wait(q_full, 0, nullptr, &never, 100000000ull);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- UMMA issuer
      bool ok = mbar_wait(q_full, 0, p.status, abort_flag);
      // descriptors of the first Q, K and V tiles; every other one is a fixed offset away
      const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024), dK = sdesc_sw128(smem_u32(sK), 16, 1024),
                     dV = sdesc_sw128(smem_u32(sV), HALF, 1024);
      auto issue_s = [&](int x, int j) {  // S_x(j) = Q_x K_j^T into TMEM columns [128 x, 128 x + 128)
        const uint64_t qd = sdesc_add(dQ, x * TILE_BYTES), kd = sdesc_add(dK, (j & 1) * TILE_BYTES);
#pragma unroll
        for (int k = 0; k < DH / 16; ++k) {
          const uint32_t off = (k >> 2) * HALF + (k & 3) * 32;
          umma_bf16_ss(tmem_base + x * 128, sdesc_add(qd, off), sdesc_add(kd, off), IDESC_QK, k != 0 ? 1u : 0u);
        }
        umma_commit(&s_full[x]);
      };
      auto issue_pv = [&](int x, int j) {  // O_x (+)= P_x(j) V_j, P_x from TMEM over S_x
        const uint64_t vd = sdesc_add(dV, (j & 1) * TILE_BYTES);
#pragma unroll
        for (int k = 0; k < BKV / 16; ++k)
          umma_bf16_ts(tmem_base + 256 + x * 128, tmem_base + x * 128 + k * 8, sdesc_add(vd, k * 16 * 128), IDESC_PV,
                       (j | k) != 0 ? 1u : 0u);
        umma_commit(&o_done[x]);
      };
      if (ok && n > 0) {
        ok = mbar_wait(&k_full[0], 0, p.status, abort_flag);
        if (ok) {
          tc_fence_after();
          issue_s(0, 0);
          issue_s(1, 0);
          umma_commit(&k_empty[0]);
        }
      }
      for (int j = 0; ok && j < n; ++j) {
        const uint32_t par = j & 1;
        for (int x = 0; ok && x < 2; ++x) {
          if (!mbar_wait(&p_full[x], par, p.status, abort_flag)) { ok = false; break; }
          if (x == 0 && !mbar_wait(&v_full[j & 1], (j >> 1) & 1, p.status, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_pv(x, j);
          if (x == 1) umma_commit(&v_empty[j & 1]);
          if (j + 1 < n) {
            // S_x(j+1) overwrites the TMEM columns P_x(j) V_j reads: wait for that MMA (an
            // MMA issued behind another is not held back from writing TMEM the earlier one
            // still reads)
            if (!mbar_wait(&o_done[x], par, p.status, abort_flag)) { ok = false; break; }
            if (x == 0 && !mbar_wait(&k_full[(j + 1) & 1], ((j + 1) >> 1) & 1, p.status, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(x, j + 1);
            if (x == 1) umma_commit(&k_empty[(j + 1) & 1]);
          }
        }
      }
      umma_commit(mma_done);
      int never = 0;
      mbar_wait(mma_done, 0, nullptr, &never, 100000000ull);
    }
  } else {
    // ------------------------------------------------------------------ softmax (two groups of 8 warps)
    const int x = (warp - 2) >> 3;        // head of this group
    const int kh = ((warp - 2) >> 2) & 1;  // half of the keys and of O's columns
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int i = q0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tSx = tmem_base + x * 128 + lane_off, tOx = tmem_base + 256 + x * 128 + lane_off + kh * 64;
    constexpr float kRescaleLog2 = 8.0f;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int k0 = bl.block(j) * BKV;
      const bool need_mask =
          !((k0 + BKV - 1 <= q0) && (p.window < 0 || q0 + BQ - 1 - k0 <= p.window || k0 + BKV - 1 < p.n_meta));
      // every thread of the group takes the same steps, so the group barrier below is
      // reached by all of them (a failed wait only skips the work)
      ok = ok && __all_sync(0xffffffffu, mbar_wait(&s_full[x], j & 1, p.status, abort_flag));
      uint32_t sv[64];
      float m_half = -INFINITY;
      if (ok) {
        tc_fence_after();
        tmem_ld32(tSx + kh * 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(tSx + kh * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_wait_ld();
        if (need_mask) {
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (!visible(i, k0 + kh * 64 + e, p.n_meta, p.window)) sv[e] = __float_as_uint(-INFINITY);
        }
        m_half = row_max64(sv) * p.scale_log2;
      }
      // the row maximum over both halves; the barrier also orders this half's reads of
      // S before the other half's P stores (P of keys 64..127 lands in S columns 32..63)
      float* sm_j = smax + (j & 1) * 512 + x * 256;
      sm_j[kh * 128 + r] = m_half;
      tc_fence_before();
      bar_sync_n(1 + x, 256);
      tc_fence_after();
      const float m_cand = fmaxf(sm_j[r], sm_j[128 + r]);
      if (ok) {
        const bool need = m_cand > m_used + kRescaleLog2;
        float alpha = 1.f;
        if (need) {
          alpha = ex2_approx(m_used - m_cand);  // 0 when m_used is -inf
          m_used = m_cand;
        }
        const float m_ref = (m_used == -INFINITY) ? 0.f : m_used;
        // P in bf16, packed in place over the first 32 words: keys 64 kh .. 64 kh + 63
        // into P columns 32 kh .. 32 kh + 31
        const float sum = row_exp64(sv, p.scale_log2, m_ref);
        tmem_st32(tSx + kh * 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        if (j > 0 && __any_sync(0xffffffffu, need)) {
          // rescale this half of O (every earlier P V of this head has completed: S_x(j)
          // was issued after it, and P_x V_j cannot start before p_full below)
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[16];
            tmem_ld16(tOx + c * 16, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st16(tOx + c * 16, o);
          }
        }
        tmem_wait_st();
        l = fmaf(l, alpha, sum);
      }
      tc_fence_before();
      mbar_arrive(&p_full[x]);
    }
    ok = ok && n > 0 && __all_sync(0xffffffffu, mbar_wait(&o_done[x], (n - 1) & 1, p.status, abort_flag));
    // the row sum over both halves (every thread of the group reaches this barrier)
    slsum[x * 256 + kh * 128 + r] = l;
    bar_sync_n(1 + x, 256);
    if (ok) {
      tc_fence_after();
      const float inv = 1.f / (slsum[x * 256 + r] + slsum[x * 256 + 128 + r]);
      __nv_bfloat16* orow = p.out + (static_cast<long long>(b) * p.T + i) * p.out_ld + (h0 + x) * DH + kh * 64;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t o[32];
        tmem_ld32(tOx + c * 32, o);
        tmem_wait_ld();
        if (i < p.T) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pack_bf16(__uint_as_float(o[8 * q]) * inv, __uint_as_float(o[8 * q + 1]) * inv),
                                pack_bf16(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv),
                                pack_bf16(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv),
                                pack_bf16(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn attn_encode_fn() {
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

// 3-D bf16 map over [batch][T][cols] with row stride ld elements; box = 64 cols x 128 rows x 1.
// rows_per_seq: the buffer's rows per sequence (>= T; rows past T read as zeros).
bool map_rows(CUtensorMap* m, const void* base, long long cols, long long ld, int T, int batch,
              long long rows_per_seq = 0) {
  EncodeTiledFn fn = attn_encode_fn();
  if (!fn) return false;
  if (rows_per_seq <= 0) rows_per_seq = T;
  cuuint64_t gd[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(batch)};
  cuuint64_t gs[2] = {static_cast<cuuint64_t>(ld) * 2, static_cast<cuuint64_t>(ld) * 2 * rows_per_seq};
  cuuint32_t bx[3] = {64, 128, 1}, es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gd, gs, bx, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_attention_f32(const AttnDesc& a, cudaStream_t st);

cudaError_t launch_attention(const AttnDesc& a, cudaStream_t st) {
  if (!a.bf16) return launch_attention_f32(a, st);
  if (a.q_row0 < 0) return cudaErrorInvalidValue;
  if (a.batch <= 0 || a.T <= 0 || a.q_row0 >= a.T) return cudaSuccess;
  static std::atomic<uint64_t> attr_done{0}, attr2_done{0};
  if (cudaError_t e = smem_attr_once(attn_fwd_tc, SMEM_BYTES, attr_done)) return e;
  CUtensorMap tq, tk, tv;
  if (!map_rows(&tq, a.q, static_cast<long long>(a.n_q_heads) * DH, a.q_ld, a.T, a.batch)) return cudaErrorInvalidValue;
  if (!map_rows(&tk, a.k, static_cast<long long>(a.n_kv_heads) * DH, a.kv_ld, a.T, a.batch, a.kv_rows))
    return cudaErrorInvalidValue;
  if (!map_rows(&tv, a.v, static_cast<long long>(a.n_kv_heads) * DH, a.kv_ld, a.T, a.batch, a.kv_rows))
    return cudaErrorInvalidValue;
  AttnParams p{};
  p.T = a.T;
  p.Hq = a.n_q_heads;
  p.Hkv = a.n_kv_heads;
  p.n_meta = a.n_meta;
  p.window = a.window;
  p.q_tiles = (a.T + BQ - 1) / BQ;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.out_ld = a.out_ld;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(DH));
  p.status = a.status;
  if ((a.n_q_heads / a.n_kv_heads) % 2 == 0) {  // pairs of query heads share each K/V tile
    if (cudaError_t e = smem_attr_once(attn_fwd_tc2, SMEM2_BYTES, attr2_done)) return e;
    dim3 grid(p.q_tiles - a.q_row0 / BQ, a.n_q_heads / 2, a.batch);
    return launch(attn_fwd_tc2, grid, dim3(576), SMEM2_BYTES, st, tq, tk, tv, p);
  }
  dim3 grid(p.q_tiles - a.q_row0 / BQ, a.n_q_heads, a.batch);
  return launch(attn_fwd_tc, grid, dim3(192), SMEM_BYTES, st, tq, tk, tv, p);
}

}  // namespace hy
