// options.cu -- option stages of the hybrid-head layer beyond the pages' formula.
//
//   conv_silu_kernel   Mamba's short causal depthwise convolution on the SSM heads'
//                      input, x = SiLU(b + sum_k w[c, k] X_ssm[t - (K-1) + k, c]) (the
//                      blog.outta.ai review, "Design formulation", names the SSM head a
//                      Mamba head; the pages print no convolution): one thread per 8
//                      channels of a 64-row run of one sequence, the last K-1 rows kept in
//                      registers, 16-byte loads and stores.
//   ssm_skip_kernel    Mamba's D skip, Y_ssm += gate * D * x, on the scan's output columns.
//   group_norm_kernel  the branch norm per group of g features (the intra-layer hybrid
//                      study on the gist.science page favours group normalisation), with
//                      beta, and the SSM half negated for difference fusion; one warp per
//                      (row, group), in place.
#include "hy_common.cuh"
#include "hy_kernels.h"

namespace hy {
namespace {

constexpr int kRun = 64;   // rows per thread of the convolution

template <typename T> struct V8;
template <> struct V8<__nv_bfloat16> {
  static HY_DEV void ld(const __nv_bfloat16* p, float (&f)[8]) {
    const uint4 q = *reinterpret_cast<const uint4*>(p);
    const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = bf16lo(u[i]);
      f[2 * i + 1] = bf16hi(u[i]);
    }
  }
  static HY_DEV void st(__nv_bfloat16* p, const float (&f)[8]) {
    *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                                              pack_bf16(f[6], f[7]));
  }
};
template <> struct V8<float> {
  static HY_DEV void ld(const float* p, float (&f)[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
  static HY_DEV void st(float* p, const float (&f)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
  }
};

template <typename T, int K>
__global__ void __launch_bounds__(256) conv_silu_kernel(const T* __restrict__ x, const T* __restrict__ w,
                                                        const float* __restrict__ bias, T* __restrict__ y, int Tseq,
                                                        int Di, int runs) {
  pdl_trigger();
  pdl_wait();
  const int cg = blockIdx.x * blockDim.x + threadIdx.x;   // 8-channel group
  if (cg * 8 >= Di) return;
  const int run = blockIdx.y % runs, b = blockIdx.y / runs;
  const int c0 = cg * 8, t0 = run * kRun, t1 = min(Tseq, t0 + kRun);
  float wk[K][8], bb[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    bb[e] = bias[c0 + e];
#pragma unroll
    for (int k = 0; k < K; ++k) wk[k][e] = to_f<T>(w[static_cast<long long>(c0 + e) * K + k]);
  }
  const long long base = static_cast<long long>(b) * Tseq;
  float hist[K][8];   // rows t - (K-1) .. t; rows before the sequence start read as zero
#pragma unroll
  for (int k = 0; k < K - 1; ++k) {
    const int t = t0 - (K - 1) + k;
#pragma unroll
    for (int e = 0; e < 8; ++e) hist[k][e] = 0.f;
    if (t >= 0) V8<T>::ld(x + (base + t) * Di + c0, hist[k]);
  }
  for (int t = t0; t < t1; ++t) {
    V8<T>::ld(x + (base + t) * Di + c0, hist[K - 1]);
    float o[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float a = bb[e];
#pragma unroll
      for (int k = 0; k < K; ++k) a = fmaf(wk[k][e], hist[k][e], a);
      o[e] = silu_f(a);
    }
    V8<T>::st(y + (base + t) * Di + c0, o);
#pragma unroll
    for (int k = 0; k < K - 1; ++k)
#pragma unroll
      for (int e = 0; e < 8; ++e) hist[k][e] = hist[k + 1][e];
  }
}

template <typename T>
__global__ void __launch_bounds__(256) ssm_skip_kernel(T* __restrict__ z, long long z_ld, const T* __restrict__ gate,
                                                       const T* __restrict__ x, const float* __restrict__ D,
                                                       long long rows, int Di) {
  pdl_trigger();
  pdl_wait();
  const int per_row = Di / 8;
  const long long total = rows * per_row;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / per_row;
    const int c = static_cast<int>(i - r * per_row) * 8;
    float zz[8], g[8], xv[8];
    V8<T>::ld(z + r * z_ld + c, zz);
    V8<T>::ld(gate + r * Di + c, g);
    V8<T>::ld(x + r * Di + c, xv);
#pragma unroll
    for (int e = 0; e < 8; ++e) zz[e] = fmaf(g[e] * D[c + e], xv[e], zz[e]);
    V8<T>::st(z + r * z_ld + c, zz);
  }
}

// One warp per (row, group of 32 * EPL features); the row's groups in order, the SSM
// half (columns >= wa) scaled by s2 (-1: difference fusion).
template <typename T, int EPL>
__global__ void __launch_bounds__(256) group_norm_kernel(T* __restrict__ z, long long rows, int wa, int ws,
                                                         const float* __restrict__ beta1,
                                                         const float* __restrict__ beta2, float s2, float eps) {
  pdl_trigger();
  pdl_wait();
  constexpr int G = 32 * EPL;
  const int W = wa + ws, groups = W / G;
  const long long wid = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= rows * groups) return;
  const long long r = wid / groups;
  const int c0 = static_cast<int>(wid - r * groups) * G + lane * EPL;
  T* p = z + r * W + c0;
  float v[EPL];
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    v[e] = to_f<T>(p[e]);
    ss = fmaf(v[e], v[e], ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const bool attn = c0 < wa;
  const float sc = rsqrtf(ss / G + eps) * (attn ? 1.f : s2);
  const float* beta = attn ? beta1 + c0 : beta2 + (c0 - wa);
#pragma unroll
  for (int e = 0; e < EPL; ++e) p[e] = from_f<T>(v[e] * sc * beta[e]);
}

}  // namespace

cudaError_t launch_conv_silu(const void* x, const void* w, const float* bias, void* y, int batch, int Tseq, int Di,
                             int K, bool bf16, cudaStream_t st) {
  if (batch <= 0 || Tseq <= 0) return cudaSuccess;
  if (Di % 8 || K < 1 || K > 4) return cudaErrorInvalidValue;
  const int runs = (Tseq + kRun - 1) / kRun;
  dim3 grid((Di / 8 + 127) / 128, batch * runs);
  const dim3 block(128);
#define HY_CONV(TT, KK)                                                                                              \
  return launch(conv_silu_kernel<TT, KK>, grid, block, 0, st, static_cast<const TT*>(x), static_cast<const TT*>(w), \
                bias, static_cast<TT*>(y), Tseq, Di, runs)
  if (bf16) {
    switch (K) {
      case 1: HY_CONV(__nv_bfloat16, 1);
      case 2: HY_CONV(__nv_bfloat16, 2);
      case 3: HY_CONV(__nv_bfloat16, 3);
      default: HY_CONV(__nv_bfloat16, 4);
    }
  }
  switch (K) {
    case 1: HY_CONV(float, 1);
    case 2: HY_CONV(float, 2);
    case 3: HY_CONV(float, 3);
    default: HY_CONV(float, 4);
  }
#undef HY_CONV
}

cudaError_t launch_ssm_skip(void* z, long long z_ld, const void* gate, const void* x, const float* D, long long rows,
                            int Di, bool bf16, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (Di % 8) return cudaErrorInvalidValue;
  const long long total = rows * (Di / 8);
  const long long blocks = (total + 255) / 256;
  const dim3 grid(static_cast<unsigned>(blocks < 8 * num_sms() ? blocks : 8 * num_sms()));
  if (bf16)
    return launch(ssm_skip_kernel<__nv_bfloat16>, grid, dim3(256), 0, st, static_cast<__nv_bfloat16*>(z), z_ld,
                  static_cast<const __nv_bfloat16*>(gate), static_cast<const __nv_bfloat16*>(x), D, rows, Di);
  return launch(ssm_skip_kernel<float>, grid, dim3(256), 0, st, static_cast<float*>(z), z_ld,
                static_cast<const float*>(gate), static_cast<const float*>(x), D, rows, Di);
}

cudaError_t launch_group_norm(void* z, long long rows, int wa, int ws, int group, const float* beta1,
                              const float* beta2, float s2, float eps, bool bf16, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if ((group != 64 && group != 128 && group != 256) || wa % group || ws % group) return cudaErrorInvalidValue;
  const long long warps = rows * ((wa + ws) / group);
  const dim3 grid(static_cast<unsigned>((warps + 7) / 8));
#define HY_GN(TT, E)                                                                                               \
  return launch(group_norm_kernel<TT, E>, grid, dim3(256), 0, st, static_cast<TT*>(z), rows, wa, ws, beta1, beta2, \
                s2, eps)
  if (bf16) {
    if (group == 64) HY_GN(__nv_bfloat16, 2);
    if (group == 128) HY_GN(__nv_bfloat16, 4);
    HY_GN(__nv_bfloat16, 8);
  }
  if (group == 64) HY_GN(float, 2);
  if (group == 128) HY_GN(float, 4);
  HY_GN(float, 8);
#undef HY_GN
}

}  // namespace hy
