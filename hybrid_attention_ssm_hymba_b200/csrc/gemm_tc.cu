// gemm_tc.cu -- bf16 GEMM C = A W^T on the sm_100a tensor cores (tcgen05.mma, fp32
// accumulators in TMEM), operands staged by TMA with 128-byte swizzle, no cluster
// multicast.  Used for the fused in_proj W_in_proj = [W_Q, W_K, W_V, W_SSM, W_G],
// x_proj, dt_proj and out_proj of the hybrid-head layer, and the SwiGLU FFN of the
// stacked blocks (blog.outta.ai Hymba review, "Design formulation"; metaphor-xennon
// page, "层配置": intermediate_size).
//
// Kernel shape: persistent, one CTA per SM, 576 threads:
//   warp 0       TMA producer (one thread) -> STAGES-deep smem ring (full/empty mbarriers)
//   warp 1       TMEM allocator + UMMA issuer (one thread), 128 x BN x 16 per instruction
//   warps 2..17  epilogue: four warps per TMEM lane quadrant, each taking every fourth
//                32-column chunk: tcgen05.ld of its chunks (all issued before the wait),
//                fused elementwise op, vector stores.  Two TMEM accumulators so the
//                epilogue of tile i overlaps the mainloop of tile i+1; sixteen warps so
//                that short-K GEMMs (dt_proj), whose time is all epilogue, keep enough
//                independent work in flight.
//
// "Meta mode" reads the rows of X~_b = [meta; x_b] for each sequence b straight from
// the meta tokens [M, K] and the user tokens x [B, L, K]: a 128-row tile that holds
// meta rows gets them from the meta tensor map and the rest from x, into the same
// swizzled smem tile, so the meta prepend costs no copy.
#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "hy_common.cuh"
#include "hy_kernels.h"

namespace hy {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int NTHREADS = 576;       // producer warp, MMA warp, 16 epilogue warps
constexpr int EPI_THREADS = 512;
constexpr int EPI_GROUPS = 4;       // epilogue warps per TMEM lane quadrant
constexpr int kMaxBiasSmem = 4096;  // a bias vector up to this length is staged in smem once
constexpr int A_STAGE = BM * BK * 2;  // 16 KB

struct GemmParams {
  int meta_mode;
  long long a_rows;  // plain mode: rows of A
  int batch, T, n_meta;
  int m_tiles;  // per sequence (meta mode) or in total (plain mode)
  int n_tiles, k_blocks, N;
  int k_blocks1;            // > 0: concatenated K, blocks [k_blocks1, k_blocks) come from A2 / W2
  int epi;
  int nseg;
  Seg seg[kMaxSegs];
  const void* resid;
  long long resid_ld;
  void* out;
  long long out_ld;
  int resid_f32, out_f32;   // residual / output element type of EPI_RESIDUAL and the dual epilogue
  int remap_L, remap_T, remap_M;  // segment rows: r -> (r / L) T + M + r % L when remap_L > 0
  int swiglu_F;
  int bias_len;             // > 0: the (single) bias segment's vector is staged in smem
  const float* bias_src;
  int dual_k;               // > 0: fused branch norm, two accumulators split at this K block
  const float2* row_ssq;
  float inv_wa, inv_ws, eps;
  unsigned* status;
};

template <int BN>
struct Cfg {
  static constexpr int B_STAGE = BN * BK * 2;
  static constexpr int STAGE = A_STAGE + B_STAGE;
  static constexpr int STAGES = (BN == 256) ? 4 : 6;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int SMEM = STAGES * STAGE + 1024 + 256;  // + bias_len * 4 when the bias is staged
  static constexpr uint32_t IDESC = idesc_bf16(BM, BN, false, false);
};

struct TileCoord {
  int b, m, n;
};
__device__ __forceinline__ TileCoord decode_tile(const GemmParams& p, int tile) {
  TileCoord c;
  const int per_b = p.m_tiles * p.n_tiles;
  c.b = p.meta_mode ? tile / per_b : 0;
  const int r = p.meta_mode ? tile - c.b * per_b : tile;
  c.m = r / p.n_tiles;
  c.n = r - c.m * p.n_tiles;
  return c;
}

// Store 16 consecutive accumulator columns [c0, c0 + 16) of one output row.
__device__ __forceinline__ void store16(const GemmParams& p, long long row, int c0, const uint32_t* v,
                                        const float* tile_bias) {
  int s = 0;
  while (s + 1 < p.nseg && c0 >= p.seg[s].col1) ++s;
  const Seg& sg = p.seg[s];
  if (c0 < sg.col0 || c0 >= sg.col1) return;
  float f[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) f[i] = __uint_as_float(v[i]);
  if (sg.op == SEG_SILU) {
#pragma unroll
    for (int i = 0; i < 16; ++i) f[i] = silu_f(f[i]);
  } else if (sg.op == SEG_SOFTPLUS_BIAS) {
    const float4* bb = reinterpret_cast<const float4*>((tile_bias ? tile_bias : sg.bias) + (c0 - sg.col0));
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 b4 = bb[j];
      f[4 * j + 0] = softplus_f(f[4 * j + 0] + b4.x);
      f[4 * j + 1] = softplus_f(f[4 * j + 1] + b4.y);
      f[4 * j + 2] = softplus_f(f[4 * j + 2] + b4.z);
      f[4 * j + 3] = softplus_f(f[4 * j + 3] + b4.w);
    }
  }
  const long long off = row * sg.ld + (c0 - sg.col0);
  if (sg.out_f32) {
    float4* d = reinterpret_cast<float4*>(static_cast<float*>(sg.ptr) + off);
#pragma unroll
    for (int j = 0; j < 4; ++j) d[j] = make_float4(f[4 * j], f[4 * j + 1], f[4 * j + 2], f[4 * j + 3]);
  } else {
    uint4* d = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(sg.ptr) + off);
#pragma unroll
    for (int j = 0; j < 2; ++j)
      d[j] = make_uint4(pack_bf16(f[8 * j], f[8 * j + 1]), pack_bf16(f[8 * j + 2], f[8 * j + 3]),
                        pack_bf16(f[8 * j + 4], f[8 * j + 5]), pack_bf16(f[8 * j + 6], f[8 * j + 7]));
  }
}

// Eight consecutive columns of a residual row (fp32 or bf16) added into f[0..8).
__device__ __forceinline__ void add_resid8(const GemmParams& p, long long row, int col, float* f) {
  if (p.resid_f32) {
    const float4* rs = reinterpret_cast<const float4*>(static_cast<const float*>(p.resid) + row * p.resid_ld + col);
    const float4 a = rs[0], b = rs[1];
    f[0] += a.x; f[1] += a.y; f[2] += a.z; f[3] += a.w;
    f[4] += b.x; f[5] += b.y; f[6] += b.z; f[7] += b.w;
  } else {
    const uint4 q = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.resid) + row * p.resid_ld + col);
    const uint32_t qq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] += bf16lo(qq[i]);
      f[2 * i + 1] += bf16hi(qq[i]);
    }
  }
}
// Eight consecutive output columns (fp32 or bf16).
__device__ __forceinline__ void store_out8(const GemmParams& p, long long row, int col, const float* f) {
  if (p.out_f32) {
    float4* d = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * p.out_ld + col);
    d[0] = make_float4(f[0], f[1], f[2], f[3]);
    d[1] = make_float4(f[4], f[5], f[6], f[7]);
  } else {
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + row * p.out_ld + col) =
        make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
  }
}

template <int BN>
__global__ void __launch_bounds__(NTHREADS, 1)
    gemm_bf16_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAx2,
                 const __grid_constant__ CUtensorMap tmM1, const __grid_constant__ CUtensorMap tmM2,
                 const __grid_constant__ CUtensorMap tmB, const __grid_constant__ GemmParams p) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* sA = smem_raw + pad;
  uint8_t* sB = sA + C::STAGES * A_STAGE;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + C::STAGES * C::B_STAGE);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_bias = reinterpret_cast<float*>(sB + C::STAGES * C::B_STAGE + 256);  // [bias_len]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], EPI_THREADS);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  pdl_trigger();
  pdl_wait();  // barriers and TMEM are set up; from here on global memory is touched
  for (int i = threadIdx.x; i < p.bias_len; i += blockDim.x) s_bias[i] = p.bias_src[i];
  if (threadIdx.x == 0) {
    tma_prefetch(&tmA);
    tma_prefetch(&tmB);
    if (p.meta_mode) {
      tma_prefetch(&tmAx2);
      tma_prefetch(&tmM1);
      tma_prefetch(&tmM2);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int total = (p.meta_mode ? p.batch : 1) * p.m_tiles * p.n_tiles;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const TileCoord tc = decode_tile(p, tile);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, p.status, abort_flag)) {
            ok = false;
            break;
          }
          uint64_t* fb = &full[stage];
          mbar_arrive_expect_tx(fb, C::STAGE);
          const int kx = kb * BK;
          uint8_t* a_dst = sA + stage * A_STAGE;
          if (p.meta_mode) {
            const int r0 = tc.m * BM;
            int mc = p.n_meta - r0;
            mc = mc < 0 ? 0 : (mc > BM ? BM : mc);
            if (mc == BM) {
              tma_load_2d(a_dst, &tmM1, fb, kx, r0);
            } else if (mc > 0) {
              tma_load_2d(a_dst, &tmM2, fb, kx, r0);
              tma_load_3d(a_dst + mc * 128, &tmAx2, fb, kx, 0, tc.b);
            } else {
              tma_load_3d(a_dst, &tmA, fb, kx, r0 - p.n_meta, tc.b);
            }
          } else if (p.k_blocks1 > 0 && kb >= p.k_blocks1) {
            // second K segment: A2 (map in the tmAx2 slot) and W2 (map in the tmM1 slot)
            tma_load_2d(a_dst, &tmAx2, fb, (kb - p.k_blocks1) * BK, tc.m * BM);
          } else {
            tma_load_2d(a_dst, &tmA, fb, kx, tc.m * BM);
          }
          uint8_t* b_dst = sB + stage * C::B_STAGE;
          if (p.epi == EPI_SWIGLU) {
            tma_load_2d(b_dst, &tmB, fb, kx, tc.n * 128);
            tma_load_2d(b_dst + 128 * 128, &tmB, fb, kx, p.swiglu_F + tc.n * 128);
          } else if (p.k_blocks1 > 0 && kb >= p.k_blocks1) {
            tma_load_2d(b_dst, &tmM1, fb, (kb - p.k_blocks1) * BK, tc.n * BN);
          } else {
            tma_load_2d(b_dst, &tmB, fb, kx, tc.n * BN);
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {  // let our own bulk copies land before the CTA's smem goes away
        int never = 0;
        for (int s = 0; s < C::STAGES; ++s)
          if (issued & (1u << s)) mbar_wait(&full[s], (last_par >> s) & 1u, nullptr, &never, 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ UMMA issuer
      // stage descriptors are fixed offsets from the first stage's (one add per MMA)
      const uint64_t dA = sdesc_sw128(smem_u32(sA), 16, 1024), dB = sdesc_sw128(smem_u32(sB), 16, 1024);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++it) {
        // dual mode: one buffer holding both accumulators (attention K blocks, then SSM)
        const int buf = p.dual_k ? 0 : (it & 1);
        const uint32_t use = p.dual_k ? (it & 1) : ((it >> 1) & 1);
        if (!mbar_wait(&tempty[buf], use ^ 1u, p.status, abort_flag)) break;
        tc_fence_after();
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          const bool second = p.dual_k && kb >= p.dual_k;
          const uint32_t d_tmem = tmem_base + (p.dual_k ? (second ? BN : 0) : buf * BN);
          const int kfirst = second ? p.dual_k : 0;  // first K block of this accumulator
          if (!mbar_wait(&full[stage], phase, p.status, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sdesc_add(dA, stage * A_STAGE), bd = sdesc_add(dB, stage * C::B_STAGE);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_bf16_ss(d_tmem, sdesc_add(ad, k * 32), sdesc_add(bd, k * 32), C::IDESC,
                         (kb != kfirst || k != 0) ? 1u : 0u);
          umma_commit(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[buf]);
      }
      umma_commit(mma_done);  // all our MMAs finished before TMEM is freed
      int never = 0;
      mbar_wait(mma_done, 0, nullptr, &never, 100000000ull);
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2..17)
    const int quad = warp & 3;          // TMEM lane quadrant this warp may access
    const int grp = (warp - 2) >> 2;    // which every-fourth 32-column chunks it takes
    const int r = quad * 32 + lane;
    constexpr int CPT = BN / 32 / EPI_GROUPS;  // chunks per thread (BN = 256: 2, BN = 128: 1)
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      const int buf = p.dual_k ? 0 : (it & 1);
      const uint32_t use = p.dual_k ? (it & 1) : ((it >> 1) & 1);
      // warp-uniform exit: tcgen05.ld below is a warp-collective instruction
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], use, p.status, abort_flag))) break;
      tc_fence_after();
      const TileCoord tc = decode_tile(p, tile);
      long long grow;
      bool valid;
      if (p.meta_mode) {
        const int t = tc.m * BM + r;
        valid = t < p.T;
        grow = static_cast<long long>(tc.b) * p.T + t;
      } else {
        grow = static_cast<long long>(tc.m) * BM + r;
        valid = grow < p.a_rows;
      }
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + buf * BN;
      if (p.dual_k) {
        // fused branch norm: out (+ resid) = rsqrt(ssq_a / wa + eps) acc_a + rsqrt(ssq_s / ws + eps) acc_s
        float sa = 0.f, ss = 0.f;
        if (valid) {
          const float2 q2 = p.row_ssq[grow];
          sa = rsqrtf(fmaf(q2.x, p.inv_wa, p.eps));
          ss = rsqrtf(fmaf(q2.y, p.inv_ws, p.eps));
        }
#pragma unroll
        for (int q = 0; q < CPT; ++q) {
          const int cc = (grp + q * EPI_GROUPS) * 32;
          uint32_t va[32], vs[32];
          tmem_ld32(tb + cc, va);
          tmem_ld32(tb + BN + cc, vs);
          tmem_wait_ld();
          if (q == CPT - 1) {
            tc_fence_before();
            mbar_arrive(&tempty[buf]);
          }
          const int col = tc.n * BN + cc;
          if (valid && col < p.N) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float f[8];
#pragma unroll
              for (int e = 0; e < 8; ++e)
                f[e] = fmaf(sa, __uint_as_float(va[8 * j + e]), ss * __uint_as_float(vs[8 * j + e]));
              if (p.epi == EPI_RESIDUAL) add_resid8(p, grow, col + 8 * j, f);
              store_out8(p, grow, col + 8 * j, f);
            }
          }
        }
        continue;
      }
      if (p.epi == EPI_SEGMENTS) {
        if (p.remap_L) grow = (grow / p.remap_L) * p.remap_T + p.remap_M + grow % p.remap_L;
        uint32_t v[CPT][32];
#pragma unroll
        for (int q = 0; q < CPT; ++q) tmem_ld32(tb + (grp + q * EPI_GROUPS) * 32, v[q]);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&tempty[buf]);  // the accumulator is in registers: free it for tile i+2
        if (valid) {
          const float* tb_bias = p.bias_len ? s_bias : nullptr;
#pragma unroll
          for (int q = 0; q < CPT; ++q) {
            const int col = tc.n * BN + (grp + q * EPI_GROUPS) * 32;
            if (col < p.N) store16(p, grow, col, v[q], tb_bias);
            if (col + 16 < p.N) store16(p, grow, col + 16, v[q] + 16, tb_bias);
          }
        }
        continue;
      } else if (p.epi == EPI_SWIGLU) {
        uint32_t g[32], u[32];
        const int c = grp;  // one 32-column chunk of the 128 gate / 128 up columns
        tmem_ld32(tb + c * 32, g);
        tmem_ld32(tb + 128 + c * 32, u);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&tempty[buf]);
        if (valid) {
          uint4* d = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + grow * p.out_ld + tc.n * 128 + c * 32);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float f[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = silu_f(__uint_as_float(g[8 * j + i])) * __uint_as_float(u[8 * j + i]);
            d[j] = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                              pack_bf16(f[6], f[7]));
          }
        }
        continue;
      } else {  // EPI_RESIDUAL
        uint32_t v[CPT][32];
#pragma unroll
        for (int q = 0; q < CPT; ++q) tmem_ld32(tb + (grp + q * EPI_GROUPS) * 32, v[q]);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&tempty[buf]);
#pragma unroll
        for (int q = 0; q < CPT; ++q) {
          const int col = tc.n * BN + (grp + q * EPI_GROUPS) * 32;
          if (valid && col < p.N) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float f[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[q][8 * j + e]);
              add_resid8(p, grow, col + 8 * j, f);
              store_out8(p, grow, col + 8 * j, f);
            }
          }
        }
        continue;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------- CTA-pair form
// The same GEMM on CTA pairs (a cluster of 2, tcgen05.mma.cta_group::2): a pair owns a
// 256 x 256 output tile; each CTA stages its own 128 rows of A and half of the tile's
// 256 rows of W (B), and one MMA instruction issued by the pair's first CTA reads both
// CTAs' operands and writes each CTA's 128 rows x 256 columns into that CTA's TMEM.  Per SM
// the shared-memory operand traffic per MMA drops from A + B (128 + 256 rows) to
// A + B/2 (128 + 128 rows).  Roles as in the one-CTA form; the second CTA's MMA warp only
// allocates TMEM.  Barriers: the first CTA's full[s] counts both CTAs' TMA bytes; each
// CTA's empty[s] and tfull[b] are signalled by the MMA's multicast commit; tempty[b] of the
// first CTA counts one arrival per epilogue warp of both CTAs.  No TMA multicast.
constexpr int PAIR_STAGES = 6;
constexpr int PAIR_B_STAGE = 128 * BK * 2;  // 16 KB: this CTA's half of the W tile
constexpr int PAIR_STAGE = A_STAGE + PAIR_B_STAGE;
constexpr int PAIR_SMEM = PAIR_STAGES * PAIR_STAGE + 1024 + 256;
constexpr uint32_t PAIR_IDESC = idesc_bf16(256, 256, false, false);

__global__ void __launch_bounds__(NTHREADS, 1)
    gemm_bf16_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAx2,
                   const __grid_constant__ CUtensorMap tmM1, const __grid_constant__ CUtensorMap tmM2,
                   const __grid_constant__ CUtensorMap tmB, const __grid_constant__ GemmParams p) {
  constexpr int BN = 256;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* sA = smem_raw + pad;
  uint8_t* sB = sA + PAIR_STAGES * A_STAGE;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + PAIR_STAGES * PAIR_B_STAGE);
  uint64_t* empty = full + PAIR_STAGES;
  uint64_t* tfull = empty + PAIR_STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_bias = reinterpret_cast<float*>(sB + PAIR_STAGES * PAIR_B_STAGE + 256);  // [bias_len]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();   // 0: issues the MMAs
  const uint32_t pair = cluster_id_x(), n_pairs = n_clusters_x();
  if (threadIdx.x == 0) {
    for (int s = 0; s < PAIR_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * (EPI_THREADS / 32));
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 2 * BN);
    tmem_relinquish_pair();
  }
  pdl_trigger();
  // both CTAs' barriers are initialised before either CTA's copies or commits reach them
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  pdl_wait();
  for (int i = threadIdx.x; i < p.bias_len; i += blockDim.x) s_bias[i] = p.bias_src[i];
  if (threadIdx.x == 0) {
    tma_prefetch(&tmA);
    tma_prefetch(&tmB);
    if (p.meta_mode) {
      tma_prefetch(&tmAx2);
      tma_prefetch(&tmM1);
      tma_prefetch(&tmM2);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = (p.meta_mode ? p.batch : 1) * p.m_tiles * p.n_tiles;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total; tile += n_pairs) {
        const TileCoord tc = decode_tile(p, tile);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, p.status, abort_flag)) {
            ok = false;
            break;
          }
          // the first CTA's full barrier counts both CTAs' bytes
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * PAIR_STAGE);
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          const int kx = kb * BK;
          uint8_t* a_dst = sA + stage * A_STAGE;
          const int r0 = tc.m * (2 * BM) + static_cast<int>(rank) * BM;   // this CTA's 128 rows
          if (p.meta_mode) {
            int mc = p.n_meta - r0;
            mc = mc < 0 ? 0 : (mc > BM ? BM : mc);
            if (mc == BM) {
              tma_load_2d_pair(a_dst, &tmM1, fb, kx, r0);
            } else if (mc > 0) {
              tma_load_2d_pair(a_dst, &tmM2, fb, kx, r0);
              tma_load_3d_pair(a_dst + mc * 128, &tmAx2, fb, kx, 0, tc.b);
            } else {
              tma_load_3d_pair(a_dst, &tmA, fb, kx, r0 - p.n_meta, tc.b);
            }
          } else if (p.k_blocks1 > 0 && kb >= p.k_blocks1) {
            tma_load_2d_pair(a_dst, &tmAx2, fb, (kb - p.k_blocks1) * BK, r0);
          } else {
            tma_load_2d_pair(a_dst, &tmA, fb, kx, r0);
          }
          uint8_t* b_dst = sB + stage * PAIR_B_STAGE;
          if (p.epi == EPI_SWIGLU) {   // first CTA: the 128 gate rows, second: the 128 up rows
            tma_load_2d_pair(b_dst, &tmB, fb, kx, (rank ? p.swiglu_F : 0) + tc.n * 128);
          } else if (p.k_blocks1 > 0 && kb >= p.k_blocks1) {
            tma_load_2d_pair(b_dst, &tmM1, fb, (kb - p.k_blocks1) * BK, tc.n * BN + static_cast<int>(rank) * 128);
          } else {
            tma_load_2d_pair(b_dst, &tmB, fb, kx, tc.n * BN + static_cast<int>(rank) * 128);
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == PAIR_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {  // let our own bulk copies land before the CTA's smem goes away (counted on CTA 0's barrier)
        int never = 0;
        if (rank == 0)
          for (int s = 0; s < PAIR_STAGES; ++s)
            if (issued & (1u << s)) mbar_wait(&full[s], (last_par >> s) & 1u, nullptr, &never, 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------ UMMA issuer (first CTA of the pair)
      const uint64_t dA = sdesc_sw128(smem_u32(sA), 16, 1024), dB = sdesc_sw128(smem_u32(sB), 16, 1024);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total; tile += n_pairs, ++it) {
        const int buf = p.dual_k ? 0 : (it & 1);
        const uint32_t use = p.dual_k ? (it & 1) : ((it >> 1) & 1);
        if (!mbar_wait(&tempty[buf], use ^ 1u, p.status, abort_flag)) break;
        tc_fence_after();
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          const bool second = p.dual_k && kb >= p.dual_k;
          const uint32_t d_tmem = tmem_base + (p.dual_k ? (second ? BN : 0) : buf * BN);
          const int kfirst = second ? p.dual_k : 0;
          if (!mbar_wait(&full[stage], phase, p.status, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sdesc_add(dA, stage * A_STAGE), bd = sdesc_add(dB, stage * PAIR_B_STAGE);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_bf16_ss_pair(d_tmem, sdesc_add(ad, k * 32), sdesc_add(bd, k * 32), PAIR_IDESC,
                              (kb != kfirst || k != 0) ? 1u : 0u);
          umma_commit_pair_mc(&empty[stage], 0x3);
          if (++stage == PAIR_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair_mc(&tfull[buf], 0x3);
      }
      umma_commit_pair_mc(mma_done, 0x1);   // all the pair's MMAs finished before TMEM is freed
      int never = 0;
      mbar_wait(mma_done, 0, nullptr, &never, 100000000ull);
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2..17 of both CTAs)
    const int quad = warp & 3;
    const int grp = (warp - 2) >> 2;
    const int r = quad * 32 + lane;
    constexpr int CPT = BN / 32 / EPI_GROUPS;
    const uint32_t tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);
    int it = 0;
    for (int tile = pair; tile < total; tile += n_pairs, ++it) {
      const int buf = p.dual_k ? 0 : (it & 1);
      const uint32_t use = p.dual_k ? (it & 1) : ((it >> 1) & 1);
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], use, p.status, abort_flag))) break;
      tc_fence_after();
      const TileCoord tc = decode_tile(p, tile);
      long long grow;
      bool valid;
      const int row_in_tile = static_cast<int>(rank) * BM + r;
      if (p.meta_mode) {
        const int t = tc.m * (2 * BM) + row_in_tile;
        valid = t < p.T;
        grow = static_cast<long long>(tc.b) * p.T + t;
      } else {
        grow = static_cast<long long>(tc.m) * (2 * BM) + row_in_tile;
        valid = grow < p.a_rows;
      }
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + buf * BN;
      // this warp is done with the accumulator: one arrival on the first CTA's tempty[buf]
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(tempty0 + buf * 8);
      };
      if (p.dual_k) {
        float sa = 0.f, ss = 0.f;
        if (valid) {
          const float2 q2 = p.row_ssq[grow];
          sa = rsqrtf(fmaf(q2.x, p.inv_wa, p.eps));
          ss = rsqrtf(fmaf(q2.y, p.inv_ws, p.eps));
        }
#pragma unroll
        for (int q = 0; q < CPT; ++q) {
          const int cc = (grp + q * EPI_GROUPS) * 32;
          uint32_t va[32], vs[32];
          tmem_ld32(tb + cc, va);
          tmem_ld32(tb + BN + cc, vs);
          tmem_wait_ld();
          if (q == CPT - 1) release();
          const int col = tc.n * BN + cc;
          if (valid && col < p.N) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float f[8];
#pragma unroll
              for (int e = 0; e < 8; ++e)
                f[e] = fmaf(sa, __uint_as_float(va[8 * j + e]), ss * __uint_as_float(vs[8 * j + e]));
              if (p.epi == EPI_RESIDUAL) add_resid8(p, grow, col + 8 * j, f);
              store_out8(p, grow, col + 8 * j, f);
            }
          }
        }
        continue;
      }
      if (p.epi == EPI_SEGMENTS) {
        if (p.remap_L) grow = (grow / p.remap_L) * p.remap_T + p.remap_M + grow % p.remap_L;
        uint32_t v[CPT][32];
#pragma unroll
        for (int q = 0; q < CPT; ++q) tmem_ld32(tb + (grp + q * EPI_GROUPS) * 32, v[q]);
        tmem_wait_ld();
        release();
        if (valid) {
          const float* tb_bias = p.bias_len ? s_bias : nullptr;
#pragma unroll
          for (int q = 0; q < CPT; ++q) {
            const int col = tc.n * BN + (grp + q * EPI_GROUPS) * 32;
            if (col < p.N) store16(p, grow, col, v[q], tb_bias);
            if (col + 16 < p.N) store16(p, grow, col + 16, v[q] + 16, tb_bias);
          }
        }
        continue;
      } else if (p.epi == EPI_SWIGLU) {
        uint32_t g[32], u[32];
        const int c = grp;
        tmem_ld32(tb + c * 32, g);
        tmem_ld32(tb + 128 + c * 32, u);
        tmem_wait_ld();
        release();
        if (valid) {
          uint4* d = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + grow * p.out_ld + tc.n * 128 + c * 32);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float f[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = silu_f(__uint_as_float(g[8 * j + i])) * __uint_as_float(u[8 * j + i]);
            d[j] = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                              pack_bf16(f[6], f[7]));
          }
        }
        continue;
      } else {  // EPI_RESIDUAL
        uint32_t v[CPT][32];
#pragma unroll
        for (int q = 0; q < CPT; ++q) tmem_ld32(tb + (grp + q * EPI_GROUPS) * 32, v[q]);
        tmem_wait_ld();
        release();
#pragma unroll
        for (int q = 0; q < CPT; ++q) {
          const int col = tc.n * BN + (grp + q * EPI_GROUPS) * 32;
          if (valid && col < p.N) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float f[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[q][8 * j + e]);
              add_resid8(p, grow, col + 8 * j, f);
              store_out8(p, grow, col + 8 * j, f);
            }
          }
        }
        continue;
      }
    }
  }
  // neither CTA frees its TMEM or leaves while the pair's MMAs may still use its shared
  // memory and TMEM
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 2 * BN);
  }
}

// ---------------------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// bf16 tensor map, innermost dimension first; 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
              const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[3], gs[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), gd, gs, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor maps and parameters of one GEMM: B (W) boxes of b_rows rows, output tiles of
// m_rows rows (one CTA: 128; a CTA pair: 256), n_cols columns.
cudaError_t prepare(const GemmDesc& g, int b_rows, int m_rows, int n_cols, CUtensorMap (&m)[5], GemmParams& p) {
  CUtensorMap &tmA = m[0], &tmAx2 = m[1], &tmM1 = m[2], &tmM2 = m[3], &tmB = m[4];
  const uint64_t K = static_cast<uint64_t>(g.K);
  p = GemmParams{};
  if (g.meta_mode) {
    const int M = g.n_meta, r = M % BM;
    uint64_t dx[3] = {K, static_cast<uint64_t>(g.L), static_cast<uint64_t>(g.batch)};
    uint64_t sx[2] = {K * 2, K * 2 * static_cast<uint64_t>(g.L)};
    uint32_t bx[3] = {BK, BM, 1};
    if (!make_map(&tmA, g.x, 3, dx, sx, bx)) return cudaErrorInvalidValue;
    tmAx2 = tmA;
    tmM1 = tmA;
    tmM2 = tmA;
    if (r != 0) {
      uint32_t bx2[3] = {BK, static_cast<uint32_t>(BM - r), 1};
      if (!make_map(&tmAx2, g.x, 3, dx, sx, bx2)) return cudaErrorInvalidValue;
    }
    if (M > 0) {
      uint64_t dm[2] = {K, static_cast<uint64_t>(M)};
      uint64_t sm[1] = {K * 2};
      uint32_t bm1[2] = {BK, BM};
      if (!make_map(&tmM1, g.meta, 2, dm, sm, bm1)) return cudaErrorInvalidValue;
      if (r != 0) {
        uint32_t bm2[2] = {BK, static_cast<uint32_t>(r)};
        if (!make_map(&tmM2, g.meta, 2, dm, sm, bm2)) return cudaErrorInvalidValue;
      }
    }
    p.meta_mode = 1;
    p.batch = g.batch;
    p.T = g.L + g.n_meta;
    p.n_meta = g.n_meta;
    p.m_tiles = (p.T + m_rows - 1) / m_rows;
    p.a_rows = static_cast<long long>(g.batch) * p.T;
  } else {
    uint64_t da[2] = {K, static_cast<uint64_t>(g.a_rows)};
    uint64_t sa[1] = {static_cast<uint64_t>(g.a_ld > 0 ? g.a_ld : g.K) * 2};
    uint32_t ba[2] = {BK, BM};
    if (!make_map(&tmA, g.a, 2, da, sa, ba)) return cudaErrorInvalidValue;
    tmAx2 = tmA;
    tmM1 = tmA;
    tmM2 = tmA;
    if (g.K2 > 0) {  // second K segment: A2 in the tmAx2 slot, W2 in the tmM1 slot
      const uint64_t K2 = static_cast<uint64_t>(g.K2);
      uint64_t da2[2] = {K2, static_cast<uint64_t>(g.a_rows)};
      uint64_t sa2[1] = {K2 * 2};
      if (!make_map(&tmAx2, g.a2, 2, da2, sa2, ba)) return cudaErrorInvalidValue;
      uint64_t dw2[2] = {K2, static_cast<uint64_t>(g.N)};
      uint32_t bw2[2] = {BK, static_cast<uint32_t>(b_rows)};
      if (!make_map(&tmM1, g.w2, 2, dw2, sa2, bw2)) return cudaErrorInvalidValue;
    }
    p.meta_mode = 0;
    p.batch = 1;
    p.a_rows = g.a_rows;
    p.m_tiles = static_cast<int>((g.a_rows + m_rows - 1) / m_rows);
  }
  {
    uint64_t dw[2] = {K, static_cast<uint64_t>(g.N)};
    uint64_t sw[1] = {K * 2};
    uint32_t bw[2] = {BK, static_cast<uint32_t>(g.epi == EPI_SWIGLU ? 128 : b_rows)};
    if (!make_map(&tmB, g.w, 2, dw, sw, bw)) return cudaErrorInvalidValue;
  }
  p.N = g.N;
  p.n_tiles = (g.epi == EPI_SWIGLU) ? g.swiglu_F / 128 : (g.N + n_cols - 1) / n_cols;
  p.k_blocks = (g.K + BK - 1) / BK;
  p.k_blocks1 = 0;
  if (g.K2 > 0 && !g.meta_mode && g.epi != EPI_SWIGLU && g.dual_k_blocks == 0) {
    p.k_blocks1 = p.k_blocks;
    p.k_blocks += (g.K2 + BK - 1) / BK;
  }
  p.epi = g.epi;
  p.nseg = g.nseg;
  p.bias_len = 0;
  p.bias_src = nullptr;
  int n_bias = 0;
  for (int i = 0; i < g.nseg; ++i) {
    p.seg[i] = g.seg[i];
    if (g.seg[i].op == SEG_SOFTPLUS_BIAS) {
      ++n_bias;
      p.bias_len = g.seg[i].col1 - g.seg[i].col0;
      p.bias_src = g.seg[i].bias;
    }
  }
  if (n_bias != 1 || p.bias_len > kMaxBiasSmem) p.bias_len = 0;  // read from global instead
  p.dual_k = g.dual_k_blocks;
  p.row_ssq = g.row_ssq;
  p.inv_wa = g.inv_wa;
  p.inv_ws = g.inv_ws;
  p.eps = g.eps;
  p.resid = g.resid;
  p.resid_ld = g.resid_ld;
  p.out = g.out;
  p.out_ld = g.out_ld;
  p.resid_f32 = g.resid_f32 ? 1 : 0;
  p.out_f32 = g.out_f32 ? 1 : 0;
  p.remap_L = g.meta_mode ? 0 : g.remap_L;
  p.remap_T = g.remap_T;
  p.remap_M = g.remap_M;
  p.swiglu_F = g.swiglu_F;
  p.status = g.status;
  return cudaSuccess;
}

template <int BN>
cudaError_t launch_bn(const GemmDesc& g, cudaStream_t st) {
  using C = Cfg<BN>;
  static std::atomic<uint64_t> attr_done{0};  // the attribute is per device
  if (cudaError_t e = smem_attr_once(gemm_bf16_tc<BN>, C::SMEM + kMaxBiasSmem * 4, attr_done)) return e;
  CUtensorMap m[5];
  GemmParams p;
  if (cudaError_t e = prepare(g, BN, BM, BN, m, p)) return e;
  const long long total = static_cast<long long>(p.meta_mode ? p.batch : 1) * p.m_tiles * p.n_tiles;
  if (total <= 0) return cudaSuccess;
  const int grid = static_cast<int>(total < num_sms() ? total : num_sms());
  return launch(gemm_bf16_tc<BN>, dim3(grid), dim3(NTHREADS), C::SMEM + p.bias_len * 4, st, m[0], m[1], m[2], m[3],
                m[4], p);
}

// The CTA-pair form: clusters of 2, as many pairs as fit at once (persistent).
cudaError_t launch_pair(const GemmDesc& g, cudaStream_t st) {
  static std::atomic<uint64_t> attr_done{0};
  if (cudaError_t e = smem_attr_once(gemm_bf16_pair, PAIR_SMEM + kMaxBiasSmem * 4, attr_done)) return e;
  CUtensorMap m[5];
  GemmParams p;
  if (cudaError_t e = prepare(g, 128, 2 * BM, 256, m, p)) return e;
  const long long total = static_cast<long long>(p.meta_mode ? p.batch : 1) * p.m_tiles * p.n_tiles;
  if (total <= 0) return cudaSuccess;
  const size_t smem = PAIR_SMEM + p.bias_len * 4;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(NTHREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  static int max_pairs[64] = {};   // pairs that fit at once, per device
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev)) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (max_pairs[dev] == 0) {
    cfg.gridDim = dim3(2 * (num_sms() / 2));
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_bf16_pair, &cfg) != cudaSuccess || n <= 0) n = num_sms() / 2;
    max_pairs[dev] = n;
  }
  const long long pairs = total < max_pairs[dev] ? total : max_pairs[dev];
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  return cudaLaunchKernelEx(&cfg, gemm_bf16_pair, m[0], m[1], m[2], m[3], m[4], p);
}

}  // namespace

// The CTA-pair GEMM is used where HYMBA_GEMM_PAIR=1 in the environment (read once).
bool use_pair_gemm() {
  static const bool on = [] {
    const char* v = std::getenv("HYMBA_GEMM_PAIR");
    return v && v[0] == '1';
  }();
  return on;
}

cudaError_t launch_gemm_bf16(const GemmDesc& g, cudaStream_t st) {
  if (g.K2 > 0 && (g.meta_mode || g.epi == EPI_SWIGLU || g.dual_k_blocks > 0 || !g.a2 || !g.w2))
    return cudaErrorInvalidValue;  // the second K segment is a plain-mode option
  if (use_pair_gemm() && (g.epi == EPI_SWIGLU || g.N > 128 || g.dual_k_blocks > 0)) return launch_pair(g, st);
  if (g.epi == EPI_SWIGLU || g.N > 128 || g.dual_k_blocks > 0) return launch_bn<256>(g, st);
  return launch_bn<128>(g, st);
}

int num_sms() {
  int dev = 0;
  cudaGetDevice(&dev);
  static int cache[64] = {0};
  if (dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

}  // namespace hy
