// decode.cu -- one generation step of the hybrid-head layer: a new token per sequence
// at row `pos` (meta rows included), from the attention heads' K/V cache and the SSM
// heads' state (blog.outta.ai Hymba review, "Efficiency and KV cache optimization": the
// SSM heads carry a fixed-size state where attention keeps a growing cache; "Combine
// global and local attention" and "Meta Tokens" for which cached rows a query sees).
//
//   attn_decode_kernel   one query row per (sequence, query head) against the visible
//                        cached keys (meta rows, then the window up to pos), split over
//                        CTAs along the keys; the query heads of one KV head share every
//                        K/V row read.  A warp takes 32 keys at a time: lane = key for the
//                        scores (its K row against the queries held in shared memory),
//                        lane = head-dim slice for P V (coalesced V rows); online softmax
//                        in fp32 (exp2 with the log2(e)/sqrt(dh) scale folded into q).
//   attn_decode_combine  merges the splits' (max, sum, unnormalised output) per row.
//   scan_step_kernel     h <- exp(A dt) h + dt x B, y = gate * (C . h) for one row, the
//                        state read and written in place; 8 lanes per channel, each with
//                        every eighth 16-byte chunk of the state.
#include "hy_common.cuh"
#include "hy_kernels.h"

namespace hy {
namespace {

constexpr int kMaxG = 8;      // query heads per KV head handled by one CTA
constexpr int kMaxEPL = 4;    // head-dim elements per lane (dh <= 128)
constexpr int kDecWarps = 4;

template <typename T> HY_DEV void load_row_f(const T* p, int n, float* f);
template <> HY_DEV void load_row_f<float>(const float* p, int n, float* f) {
  for (int i = 0; i < n; i += 4) {
    const float4 v = *reinterpret_cast<const float4*>(p + i);
    f[i] = v.x; f[i + 1] = v.y; f[i + 2] = v.z; f[i + 3] = v.w;
  }
}
template <> HY_DEV void load_row_f<__nv_bfloat16>(const __nv_bfloat16* p, int n, float* f) {
  for (int i = 0; i < n; i += 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(p + i);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f[i + 2 * k] = bf16lo(u[k]);
      f[i + 2 * k + 1] = bf16hi(u[k]);
    }
  }
}

struct DecodeAttnParams {
  const void* q;            // [B, Hq*dh]
  const void* k;            // [B, cap, kv_ld] (row pos of sequence b at (b*cap + pos)*kv_ld)
  const void* v;
  long long cap, kv_ld;
  float* part;              // [B, Hq, splits, dh + 2]: unnormalised o, then (max, sum) in log2 units
  int Hq, Hkv, dh, pos, n_meta, window, splits, keys_per_split;
  float scale_log2;
};

// Visible keys of the query at `pos`, in order: meta rows below the window, then the
// window [w_lo, pos] (global attention: [0, pos]).
struct VisKeys {
  int m_cnt, w_lo, n;
  HY_DEV int key(int idx) const { return idx < m_cnt ? idx : w_lo + (idx - m_cnt); }
};
HY_DEV VisKeys vis_keys(int pos, int n_meta, int window) {
  VisKeys v;
  v.w_lo = window < 0 ? 0 : max(0, pos - window);
  v.m_cnt = min(n_meta, v.w_lo);
  v.n = v.m_cnt + (pos - v.w_lo + 1);
  return v;
}

template <typename T>
__global__ void __launch_bounds__(32 * kDecWarps) attn_decode_kernel(const DecodeAttnParams p) {
  pdl_trigger();
  pdl_wait();
  __shared__ float sq[kMaxG][128];
  __shared__ float s_m[kDecWarps][kMaxG], s_l[kDecWarps][kMaxG];
  __shared__ float s_o[kDecWarps][kMaxG][128];
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int G = p.Hq / p.Hkv, dh = p.dh, epl = dh / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* qb = static_cast<const T*>(p.q) + static_cast<long long>(b) * p.Hq * dh + static_cast<long long>(kvh) * G * dh;
  for (int i = threadIdx.x; i < G * dh; i += blockDim.x) sq[i / dh][i % dh] = to_f<T>(qb[i]) * p.scale_log2;
  __syncthreads();
  const VisKeys vk = vis_keys(p.pos, p.n_meta, p.window);
  const int k0 = split * p.keys_per_split, k1 = min(vk.n, k0 + p.keys_per_split);
  const T* kb = static_cast<const T*>(p.k) + static_cast<long long>(b) * p.cap * p.kv_ld + kvh * dh;
  const T* vb = static_cast<const T*>(p.v) + static_cast<long long>(b) * p.cap * p.kv_ld + kvh * dh;
  float m[kMaxG], l[kMaxG], o[kMaxG][kMaxEPL];
#pragma unroll
  for (int g = 0; g < kMaxG; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < kMaxEPL; ++e) o[g][e] = 0.f;
  }
  for (int c0 = k0 + warp * 32; c0 < k1; c0 += 32 * kDecWarps) {
    const int idx = c0 + lane;
    const bool valid = idx < k1;
    // scores: lane = key
    float s[kMaxG];
#pragma unroll
    for (int g = 0; g < kMaxG; ++g) s[g] = 0.f;
    if (valid) {
      const T* kr = kb + static_cast<long long>(vk.key(idx)) * p.kv_ld;
      if constexpr (sizeof(T) == 2) {
        // the whole K row (dh <= 128: at most 16 vectors) in flight before any is used
        uint4 kv[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (8 * j < dh) kv[j] = *reinterpret_cast<const uint4*>(kr + 8 * j);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (8 * j >= dh) continue;
          const uint32_t u[4] = {kv[j].x, kv[j].y, kv[j].z, kv[j].w};
          float kf[8];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            kf[2 * q] = bf16lo(u[q]);
            kf[2 * q + 1] = bf16hi(u[q]);
          }
#pragma unroll
          for (int g = 0; g < kMaxG; ++g) {
            if (g < G) {
#pragma unroll
              for (int e = 0; e < 8; ++e) s[g] = fmaf(sq[g][8 * j + e], kf[e], s[g]);
            }
          }
        }
      } else {
        for (int e0 = 0; e0 < dh; e0 += 8) {
          float kf[8];
          load_row_f<T>(kr + e0, 8, kf);
#pragma unroll
          for (int g = 0; g < kMaxG; ++g) {
            if (g < G) {
#pragma unroll
              for (int e = 0; e < 8; ++e) s[g] = fmaf(sq[g][e0 + e], kf[e], s[g]);
            }
          }
        }
      }
    }
    float pr[kMaxG];
#pragma unroll
    for (int g = 0; g < kMaxG; ++g) {
      if (g >= G) continue;
      float v = valid ? s[g] : -INFINITY;
      float cm = v;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
      const float mn = fmaxf(m[g], cm);   // finite: every chunk has at least one valid key
      const float sc = ex2_approx(m[g] - mn);
      pr[g] = valid ? ex2_approx(v - mn) : 0.f;
      float ps = pr[g];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l[g] = fmaf(l[g], sc, ps);
      m[g] = mn;
#pragma unroll
      for (int e = 0; e < kMaxEPL; ++e) o[g][e] *= sc;
    }
    // P V: lane = head-dim slice [lane * epl, lane * epl + epl)
    const int nk = min(32, k1 - c0);
    for (int kk0 = 0; kk0 < nk; kk0 += 8) {
      // eight V rows' slices in flight at once
      float vf[8][kMaxEPL];
#pragma unroll
      for (int u8 = 0; u8 < 8; ++u8) {
        const int kk = kk0 + u8;
        const T* vr = vb + static_cast<long long>(vk.key(c0 + min(kk, nk - 1))) * p.kv_ld + lane * epl;
#pragma unroll
        for (int e = 0; e < kMaxEPL; ++e) vf[u8][e] = e < epl ? to_f<T>(vr[e]) : 0.f;
      }
#pragma unroll
      for (int u8 = 0; u8 < 8; ++u8) {
        const int kk = kk0 + u8;
#pragma unroll
        for (int g = 0; g < kMaxG; ++g) {
          if (g >= G) continue;
          const float pk = __shfl_sync(0xffffffffu, pr[g], kk & 31);
          if (kk < nk) {
#pragma unroll
            for (int e = 0; e < kMaxEPL; ++e) o[g][e] = fmaf(pk, vf[u8][e], o[g][e]);
          }
        }
      }
    }
  }
  // merge the warps of the CTA
#pragma unroll
  for (int g = 0; g < kMaxG; ++g) {
    if (g >= G) continue;
    if (lane == 0) {
      s_m[warp][g] = m[g];
      s_l[warp][g] = l[g];
    }
#pragma unroll
    for (int e = 0; e < kMaxEPL; ++e)
      if (e < epl) s_o[warp][g][lane * epl + e] = o[g][e];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * dh; i += blockDim.x) {
    const int g = i / dh, e = i % dh;
    float mm = -INFINITY;
    for (int w = 0; w < kDecWarps; ++w) mm = fmaxf(mm, s_m[w][g]);
    float ll = 0.f, oo = 0.f;
    if (mm != -INFINITY) {
      for (int w = 0; w < kDecWarps; ++w) {
        const float sc = s_m[w][g] == -INFINITY ? 0.f : ex2_approx(s_m[w][g] - mm);
        ll = fmaf(s_l[w][g], sc, ll);
        oo = fmaf(s_o[w][g][e], sc, oo);
      }
    }
    const int h = kvh * G + g;
    float* dst = p.part + ((static_cast<long long>(b) * p.Hq + h) * p.splits + split) * (dh + 2);
    dst[e] = oo;
    if (e == 0) {
      dst[dh] = mm;
      dst[dh + 1] = ll;
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(128) attn_decode_combine(const float* __restrict__ part, T* out, long long out_ld,
                                                           int Hq, int dh, int splits) {
  pdl_trigger();
  pdl_wait();
  const int h = blockIdx.x, b = blockIdx.y;
  const float* pb = part + (static_cast<long long>(b) * Hq + h) * splits * (dh + 2);
  float mm = -INFINITY;
  for (int s = 0; s < splits; ++s) mm = fmaxf(mm, pb[s * (dh + 2) + dh]);
  for (int e = threadIdx.x; e < dh; e += blockDim.x) {
    float ll = 0.f, oo = 0.f;
    for (int s = 0; s < splits; ++s) {
      const float ms = pb[s * (dh + 2) + dh];
      if (ms == -INFINITY) continue;
      const float sc = ex2_approx(ms - mm);
      ll = fmaf(pb[s * (dh + 2) + dh + 1], sc, ll);
      oo = fmaf(pb[s * (dh + 2) + e], sc, oo);
    }
    out[static_cast<long long>(b) * out_ld + h * dh + e] = from_f<T>(oo / ll);
  }
}

// One step of the selective scan per (sequence, channel): 8 lanes per channel, N / 8 state
// components each.  a_log [Di] (one decay per channel) or [Di, N] (per channel and state).
template <typename T>
__global__ void __launch_bounds__(256) scan_step_kernel(const T* __restrict__ x, const T* __restrict__ dt,
                                                        const float* __restrict__ bc, const T* __restrict__ gate,
                                                        const float* __restrict__ a_log, int a_per_state,
                                                        float* __restrict__ h, T* __restrict__ y, long long y_ld,
                                                        int B, int Di, int N, const float* __restrict__ d_skip) {
  pdl_trigger();
  pdl_wait();
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long ch = gid >> 3;            // (b, c) pair
  const int sl = threadIdx.x & 7, ns = N / 8;
  const bool valid = ch < static_cast<long long>(B) * Di;
  const int b = valid ? static_cast<int>(ch / Di) : 0, c = valid ? static_cast<int>(ch % Di) : 0;
  float yv = 0.f;
  if (valid) {
    // lane sl owns the 16-byte chunks sl, sl + 8, ... of the channel's state (and of B, C):
    // the 8 lanes of a channel read 128 contiguous bytes per step, every load issued first
    const long long r = static_cast<long long>(b) * Di + c;
    const float d = to_f<T>(dt[r]), u = d * to_f<T>(x[r]);
    const float4* B4 = reinterpret_cast<const float4*>(bc + static_cast<long long>(b) * 2 * N);
    const float4* C4 = B4 + N / 4;
    float4* h4 = reinterpret_cast<float4*>(h + r * N);
    const float4* al4 = reinterpret_cast<const float4*>(a_log + static_cast<long long>(c) * N);
    const float A1 = a_per_state ? 0.f : -expf(a_log[c]) * 1.4426950408889634f;
    const float a1 = ex2_approx(A1 * d);
    const int nq = N / 4;
    for (int base = 0; base < nq; base += 32) {   // 128 states per pass (one pass for N <= 128)
      float4 hv[4], bv[4], cv[4], av[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int q = base + sl + 8 * i;
        if (q < nq) {
          hv[i] = h4[q];
          bv[i] = B4[q];
          cv[i] = C4[q];
          av[i] = a_per_state ? al4[q] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int q = base + sl + 8 * i;
        if (q < nq) {
          float a[4] = {a1, a1, a1, a1};
          if (a_per_state) {
            const float al[4] = {av[i].x, av[i].y, av[i].z, av[i].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) a[e] = ex2_approx(-expf(al[e]) * 1.4426950408889634f * d);
          }
          float4 hn;
          hn.x = fmaf(a[0], hv[i].x, u * bv[i].x);
          hn.y = fmaf(a[1], hv[i].y, u * bv[i].y);
          hn.z = fmaf(a[2], hv[i].z, u * bv[i].z);
          hn.w = fmaf(a[3], hv[i].w, u * bv[i].w);
          h4[q] = hn;
          yv = fmaf(cv[i].x, hn.x, fmaf(cv[i].y, hn.y, fmaf(cv[i].z, hn.z, fmaf(cv[i].w, hn.w, yv))));
        }
      }
    }
  }
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) yv += __shfl_xor_sync(0xffffffffu, yv, off);
  if (valid && sl == 0) {
    const long long r = static_cast<long long>(b) * Di + c;
    if (d_skip) yv = fmaf(d_skip[c], to_f<T>(x[r]), yv);
    y[static_cast<long long>(b) * y_ld + c] = from_f<T>(to_f<T>(gate[r]) * yv);
  }
}

}  // namespace

int decode_attn_splits(int batch, int n_kv_heads, int n_visible, int max_splits, int* keys_per_split) {
  int target = (4 * num_sms() + batch * n_kv_heads - 1) / (batch * n_kv_heads);
  if (target > max_splits) target = max_splits;   // keys_per_split >= n / target: splits <= target
  int kps = (n_visible + target - 1) / target;
  kps = ((kps + 127) / 128) * 128;   // whole 32-key chunks for every warp of the CTA
  if (kps < 128) kps = 128;
  *keys_per_split = kps;
  return (n_visible + kps - 1) / kps;
}

cudaError_t launch_attention_decode(const DecodeAttnDesc& a, cudaStream_t st) {
  if (a.head_dim % 32 || a.head_dim > 128 || a.n_q_heads / a.n_kv_heads > kMaxG) return cudaErrorInvalidValue;
  DecodeAttnParams p;
  p.q = a.q;
  p.k = a.k;
  p.v = a.v;
  p.cap = a.cap;
  p.kv_ld = a.kv_ld;
  p.part = a.part;
  p.Hq = a.n_q_heads;
  p.Hkv = a.n_kv_heads;
  p.dh = a.head_dim;
  p.pos = a.pos;
  p.n_meta = a.n_meta;
  p.window = a.window;
  const int w_lo = a.window < 0 ? 0 : (a.pos - a.window > 0 ? a.pos - a.window : 0);
  const int n_vis = (a.n_meta < w_lo ? a.n_meta : w_lo) + (a.pos - w_lo + 1);
  p.splits = decode_attn_splits(a.batch, a.n_kv_heads, n_vis, a.max_splits, &p.keys_per_split);
  if (p.splits > a.max_splits) return cudaErrorInvalidValue;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(a.head_dim));
  dim3 grid(p.splits, a.n_kv_heads, a.batch);
  cudaError_t e = a.bf16 ? launch(attn_decode_kernel<__nv_bfloat16>, grid, dim3(32 * kDecWarps), 0, st, p)
                         : launch(attn_decode_kernel<float>, grid, dim3(32 * kDecWarps), 0, st, p);
  if (e != cudaSuccess) return e;
  dim3 g2(a.n_q_heads, a.batch);
  return a.bf16 ? launch(attn_decode_combine<__nv_bfloat16>, g2, dim3(128), 0, st, static_cast<const float*>(a.part),
                         static_cast<__nv_bfloat16*>(a.out), a.out_ld, a.n_q_heads, a.head_dim, p.splits)
                : launch(attn_decode_combine<float>, g2, dim3(128), 0, st, static_cast<const float*>(a.part),
                         static_cast<float*>(a.out), a.out_ld, a.n_q_heads, a.head_dim, p.splits);
}

cudaError_t launch_scan_step(const ScanStepDesc& s, cudaStream_t st) {
  if (s.d_state % 8 || s.d_state > 256) return cudaErrorInvalidValue;
  const long long threads = static_cast<long long>(s.batch) * s.d_inner * 8;
  const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
  if (s.bf16)
    return launch(scan_step_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, st,
                  static_cast<const __nv_bfloat16*>(s.x), static_cast<const __nv_bfloat16*>(s.dt), s.bc,
                  static_cast<const __nv_bfloat16*>(s.gate), s.a_log, s.a_per_state ? 1 : 0, s.h,
                  static_cast<__nv_bfloat16*>(s.y), s.y_ld, s.batch, s.d_inner, s.d_state, s.d_skip);
  return launch(scan_step_kernel<float>, dim3(blocks), dim3(256), 0, st, static_cast<const float*>(s.x),
                static_cast<const float*>(s.dt), s.bc, static_cast<const float*>(s.gate), s.a_log,
                s.a_per_state ? 1 : 0, s.h, static_cast<float*>(s.y), s.y_ld, s.batch, s.d_inner, s.d_state,
                s.d_skip);
}

}  // namespace hy
