// norm.cu -- row-wise RMS normalisation kernels.
//
//   branch_norm: z = [beta1 * rms(z_attn) || beta2 * rms(z_ssm)] in place, the
//     per-branch norm and learnable rescale before out_proj (blog.outta.ai Hymba
//     review, "Design formulation", total fusion formulation; metaphor-xennon
//     "PyTorch伪代码": one RMSNorm per branch).
//   rmsnorm:     y = x / sqrt(mean(x^2) + eps), unit gain (pre-norm of the
//     stacked blocks).
//   row_ssq, scale_cols: the two pieces of the branch norm fused into out_proj (bf16):
//     per-row sums of squares of both branches, and W_out with beta folded into its
//     columns.
// bf16 rows up to 6144 elements: one warp per row with the row held in registers
// (one HBM read, one write).  Wider rows and fp32: one CTA per row (the second read
// of the row hits L1/L2).  fp32 sums; 16-byte vector loads and stores.  row_ssq, a pure
// read of Z, streams Z through shared memory with bulk copies (one CTA per SM).
#include <algorithm>

#include "hy_common.cuh"
#include "hy_kernels.h"

namespace hy {
namespace {

constexpr int NT = 256;

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
  if (threadIdx.x < 32) {
    s = (l < NT / 32) ? red[l] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (l == 0) red[NT / 32] = s;
  }
  __syncthreads();
  return red[NT / 32];
}

// vector of 8 elements
template <typename T> struct Vec8;
template <> struct Vec8<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&f)[8]) {
    const uint4 q = *reinterpret_cast<const uint4*>(p);
    const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = bf16lo(u[i]);
      f[2 * i + 1] = bf16hi(u[i]);
    }
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&f)[8]) {
    *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                                              pack_bf16(f[6], f[7]));
  }
};
template <> struct Vec8<float> {
  static __device__ __forceinline__ void load(const float* p, float (&f)[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&f)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
  }
};

template <typename T>
__device__ __forceinline__ float sumsq(const T* row, int w) {
  float s = 0.f;
  for (int i = threadIdx.x * 8; i < w; i += NT * 8) {
    float f[8];
    Vec8<T>::load(row + i, f);
#pragma unroll
    for (int j = 0; j < 8; ++j) s = fmaf(f[j], f[j], s);
  }
  return s;
}

template <typename T>
__device__ __forceinline__ void scale_row(const T* src, T* dst, int w, float r, const float* beta) {
  for (int i = threadIdx.x * 8; i < w; i += NT * 8) {
    float f[8];
    Vec8<T>::load(src + i, f);
    if (beta) {
      const float4 b0 = *reinterpret_cast<const float4*>(beta + i), b1 = *reinterpret_cast<const float4*>(beta + i + 4);
      const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) f[j] = f[j] * r * bb[j];
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) f[j] *= r;
    }
    Vec8<T>::store(dst + i, f);
  }
}

template <typename T>
__global__ void __launch_bounds__(NT) branch_norm_kernel(T* z, const float* __restrict__ beta1,
                                                         const float* __restrict__ beta2, int wa, int ws, float eps,
                                                         float s2) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[NT / 32 + 1];
  T* row = z + static_cast<long long>(blockIdx.x) * (wa + ws);
  const float sa = block_sum(sumsq(row, wa), red);
  const float ss = block_sum(sumsq(row + wa, ws), red);
  const float ra = rsqrtf(sa / wa + eps), rs = rsqrtf(ss / ws + eps);
  scale_row(row, row, wa, ra, beta1);
  scale_row(row + wa, row + wa, ws, rs * s2, beta2);
}

template <typename T>
__global__ void __launch_bounds__(NT) rmsnorm_kernel(const T* x, T* y, int d, float eps) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[NT / 32 + 1];
  const long long off = static_cast<long long>(blockIdx.x) * d;
  const float s = block_sum(sumsq(x + off, d), red);
  scale_row(x + off, y + off, d, rsqrtf(s / d + eps), nullptr);
}

// bf16 rows up to 32 * 8 * MAXV elements: one warp per row, the row held in
// registers (16-byte vectors, lane-interleaved), one read and one write of HBM,
// warp-shuffle sums.  `wa` (the first branch's width) is a multiple of 8, so no
// vector straddles the two branches; wa = 0 gives a plain unit-gain RMSNorm.
template <int MAXV>
__global__ void __launch_bounds__(256) rownorm_warp_kernel(const __nv_bfloat16* x,  // x and y may alias
                                                           __nv_bfloat16* y, long long rows, int wa,
                                                           int ws, const float* __restrict__ beta1,
                                                           const float* __restrict__ beta2, float eps, float s2) {
  pdl_trigger();
  pdl_wait();
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int W = wa + ws;
  const int nv = W / 8;
  const uint4* src = reinterpret_cast<const uint4*>(x + row * W);
  uint4 v[MAXV];
  float sa = 0.f, ss = 0.f;
  // every load of the row issued before any is used (a short grid has no other warps to
  // hide their latency behind)
#pragma unroll
  for (int k = 0; k < MAXV; ++k) {
    const int vi = lane + 32 * k;
    v[k] = vi < nv ? src[vi] : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int k = 0; k < MAXV; ++k) {
    const int vi = lane + 32 * k;
    if (vi < nv) {
      const uint32_t u[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
      float acc = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float a = bf16lo(u[q]), bb = bf16hi(u[q]);
        acc = fmaf(a, a, fmaf(bb, bb, acc));
      }
      if (vi * 8 < wa) sa += acc;
      else ss += acc;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sa += __shfl_xor_sync(0xffffffffu, sa, o);
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
  }
  const float ra = wa > 0 ? rsqrtf(sa / wa + eps) : 0.f, rs = rsqrtf(ss / ws + eps);
  uint4* dst = reinterpret_cast<uint4*>(y + row * W);
#pragma unroll
  for (int k = 0; k < MAXV; ++k) {
    const int vi = lane + 32 * k;
    if (vi < nv) {
      const int col = vi * 8;
      const bool first = col < wa;
      const float r = first ? ra : rs * s2;
      const float* beta = first ? beta1 + col : (beta2 ? beta2 + (col - wa) : nullptr);
      const uint32_t u[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
      float f[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        f[2 * q] = bf16lo(u[q]) * r;
        f[2 * q + 1] = bf16hi(u[q]) * r;
      }
      if (beta) {
        const float4 b0 = *reinterpret_cast<const float4*>(beta), b1 = *reinterpret_cast<const float4*>(beta + 4);
        f[0] *= b0.x; f[1] *= b0.y; f[2] *= b0.z; f[3] *= b0.w;
        f[4] *= b1.x; f[5] *= b1.y; f[6] *= b1.z; f[7] *= b1.w;
      }
      dst[vi] = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
    }
  }
}

// The same norm for a few rows (a generation step): a CTA per row, 256 threads with at
// most MAXV 16-byte vectors each, the row and its beta values loaded before any use.
template <int MAXV>
__global__ void __launch_bounds__(256) rownorm_cta_kernel(const __nv_bfloat16* x,  // x and y may alias
                                                          __nv_bfloat16* y, int wa, int ws,
                                                          const float* __restrict__ beta1,
                                                          const float* __restrict__ beta2, float eps, float s2) {
  __shared__ float red[8][2];
  pdl_trigger();
  pdl_wait();
  const long long row = blockIdx.x;
  const int W = wa + ws, nv = W / 8;
  const uint4* src = reinterpret_cast<const uint4*>(x + row * W);
  uint4 v[MAXV];
  float4 bl[MAXV], bh[MAXV];
#pragma unroll
  for (int k = 0; k < MAXV; ++k) {
    const int vi = threadIdx.x + 256 * k;
    v[k] = make_uint4(0u, 0u, 0u, 0u);
    bl[k] = bh[k] = make_float4(1.f, 1.f, 1.f, 1.f);
    if (vi < nv) {
      v[k] = src[vi];
      const int col = vi * 8;
      const float* beta = col < wa ? beta1 + col : (beta2 ? beta2 + (col - wa) : nullptr);
      if (beta) {
        bl[k] = *reinterpret_cast<const float4*>(beta);
        bh[k] = *reinterpret_cast<const float4*>(beta + 4);
      }
    }
  }
  float sa = 0.f, ss = 0.f;
#pragma unroll
  for (int k = 0; k < MAXV; ++k) {
    const int vi = threadIdx.x + 256 * k;
    const uint32_t u[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
    float acc = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float a = bf16lo(u[q]), bb = bf16hi(u[q]);
      acc = fmaf(a, a, fmaf(bb, bb, acc));
    }
    if (vi * 8 < wa) sa += acc;
    else ss += acc;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sa += __shfl_xor_sync(0xffffffffu, sa, o);
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    red[warp][0] = sa;
    red[warp][1] = ss;
  }
  __syncthreads();
  sa = ss = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    sa += red[w][0];
    ss += red[w][1];
  }
  const float ra = wa > 0 ? rsqrtf(sa / wa + eps) : 0.f, rs = rsqrtf(ss / ws + eps);
  uint4* dst = reinterpret_cast<uint4*>(y + row * W);
#pragma unroll
  for (int k = 0; k < MAXV; ++k) {
    const int vi = threadIdx.x + 256 * k;
    if (vi < nv) {
      const float r = vi * 8 < wa ? ra : rs * s2;
      const uint32_t u[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
      const float b[8] = {bl[k].x, bl[k].y, bl[k].z, bl[k].w, bh[k].x, bh[k].y, bh[k].z, bh[k].w};
      float f[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        f[2 * q] = bf16lo(u[q]) * r * b[2 * q];
        f[2 * q + 1] = bf16hi(u[q]) * r * b[2 * q + 1];
      }
      dst[vi] = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
    }
  }
}

template <int MAXV>
void launch_rownorm(const void* x, void* y, long long rows, int wa, int ws, const float* b1, const float* b2,
                    float eps, float s2, cudaStream_t st) {
  launch(rownorm_warp_kernel<MAXV>, dim3(static_cast<unsigned>((rows + 7) / 8)), dim3(256), 0, st,
         static_cast<const __nv_bfloat16*>(x), static_cast<__nv_bfloat16*>(y), rows, wa, ws, b1, b2, eps, s2);
}

// picks the smallest register footprint that holds a row; false if the row is too wide
bool rownorm_bf16(const void* x, void* y, long long rows, int wa, int ws, const float* b1, const float* b2, float eps,
                  cudaStream_t st, float s2 = 1.f) {
  const int nv = (wa + ws) / 8;
  if (rows < 512 && nv <= 4 * 256) {   // too few rows to fill the GPU one warp each
    const auto args = [&](auto kern) {
      launch(kern, dim3(static_cast<unsigned>(rows)), dim3(256), 0, st, static_cast<const __nv_bfloat16*>(x),
             static_cast<__nv_bfloat16*>(y), wa, ws, b1, b2, eps, s2);
    };
    if (nv <= 256) args(rownorm_cta_kernel<1>);
    else if (nv <= 512) args(rownorm_cta_kernel<2>);
    else if (nv <= 768) args(rownorm_cta_kernel<3>);
    else args(rownorm_cta_kernel<4>);
    return true;
  }
  const int per_lane = (nv + 31) / 32;
  if (per_lane <= 4) launch_rownorm<4>(x, y, rows, wa, ws, b1, b2, eps, s2, st);
  else if (per_lane <= 8) launch_rownorm<8>(x, y, rows, wa, ws, b1, b2, eps, s2, st);
  else if (per_lane <= 12) launch_rownorm<12>(x, y, rows, wa, ws, b1, b2, eps, s2, st);
  else if (per_lane <= 16) launch_rownorm<16>(x, y, rows, wa, ws, b1, b2, eps, s2, st);
  else if (per_lane <= 24) launch_rownorm<24>(x, y, rows, wa, ws, b1, b2, eps, s2, st);
  else return false;
  return true;
}

// Row sums of squares of the two branches of Z (bf16), one warp per row, the row held
// in registers (16-byte vectors): ssq[row] = (sum over [0, wa), sum over [wa, wa + ws)).
// wa is a multiple of 8, so no vector straddles the branches.
template <int MAXV>
__global__ void __launch_bounds__(256) row_ssq_kernel(const __nv_bfloat16* __restrict__ z, long long rows, int wa,
                                                      int ws, float2* __restrict__ ssq) {
  pdl_trigger();
  pdl_wait();
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int nv = (wa + ws) / 8;
  const uint4* src = reinterpret_cast<const uint4*>(z + row * (wa + ws));
  uint4 v[MAXV];
#pragma unroll
  for (int k = 0; k < MAXV; ++k)
    if (lane + 32 * k < nv) v[k] = src[lane + 32 * k];
  float sa = 0.f, ss = 0.f;
#pragma unroll
  for (int k = 0; k < MAXV; ++k) {
    const int vi = lane + 32 * k;
    if (vi < nv) {
      const uint32_t u[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
      float acc = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) acc = fmaf(bf16lo(u[q]), bf16lo(u[q]), fmaf(bf16hi(u[q]), bf16hi(u[q]), acc));
      if (vi * 8 < wa) sa += acc;
      else ss += acc;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sa += __shfl_xor_sync(0xffffffffu, sa, o);
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
  }
  if (lane == 0) ssq[row] = make_float2(sa, ss);
}

// The same sums with Z streamed through shared memory by bulk copies.  Z's rows are
// contiguous, so a chunk of rpc rows is one copy; one CTA per SM walks chunks blockIdx.x,
// blockIdx.x + gridDim.x, ... through a ring of nst chunks: warp 8 (one thread) issues the
// copies, warps 0..7 take the chunk's rows (row w, w + 8, ...) and reduce them from shared
// memory.  The copy engine keeps more bytes in flight per SM than the warps' own 16-byte
// loads can, which a stream over HBM needs.
constexpr int SSQ_WARPS = 8;
constexpr int SSQ_RING = 200 * 1024;   // bytes of the ring at most

__global__ void __launch_bounds__((SSQ_WARPS + 1) * 32, 1)
    row_ssq_bulk_kernel(const __nv_bfloat16* __restrict__ z, long long rows, int wa, int ws, int rpc, int nst,
                        float2* __restrict__ ssq, unsigned* status) {
  extern __shared__ __align__(16) uint8_t ring[];  // [nst][rpc rows], then full[nst], empty[nst], abort flag
  const uint32_t row_bytes = static_cast<uint32_t>(wa + ws) * 2u, chunk_bytes = row_bytes * rpc;
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + static_cast<size_t>(nst) * chunk_bytes);
  uint64_t* empty = full + nst;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + nst);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long nchunk = (rows + rpc - 1) / rpc;
  if (threadIdx.x == 0) {
    for (int s = 0; s < nst; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], SSQ_WARPS);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();
  if (warp == SSQ_WARPS) {
    if (lane == 0) {
      long long i = 0;  // chunks issued
      for (long long q = blockIdx.x; q < nchunk; q += gridDim.x, ++i) {
        const int s = static_cast<int>(i % nst);
        if (i >= nst && !mbar_wait(&empty[s], static_cast<uint32_t>((i / nst) - 1) & 1u, status, abort_flag)) break;
        const long long r0 = q * rpc;
        const uint32_t bytes = static_cast<uint32_t>(rows - r0 < rpc ? rows - r0 : rpc) * row_bytes;
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_load_1d(ring + static_cast<size_t>(s) * chunk_bytes, reinterpret_cast<const uint8_t*>(z) + r0 * row_bytes,
                     bytes, &full[s]);
      }
      // the copies still in flight land before shared memory goes away
      int never = 0;
      for (long long j = (i > nst ? i - nst : 0); j < i; ++j)
        mbar_wait(&full[j % nst], static_cast<uint32_t>(j / nst) & 1u, nullptr, &never, 100000000ull);
    }
  } else {
    const int nva = wa / 8, nv = (wa + ws) / 8;
    long long i = 0;
    for (long long q = blockIdx.x; q < nchunk; q += gridDim.x, ++i) {
      const int s = static_cast<int>(i % nst);
      if (!mbar_wait(&full[s], static_cast<uint32_t>(i / nst) & 1u, status, abort_flag)) break;
      const long long r0 = q * rpc;
      const int nr = static_cast<int>(rows - r0 < rpc ? rows - r0 : rpc);
      for (int r = warp; r < nr; r += SSQ_WARPS) {
        const uint32_t base = smem_u32(ring + static_cast<size_t>(s) * chunk_bytes + static_cast<size_t>(r) * row_bytes);
        float sa = 0.f, ss = 0.f;
#pragma unroll 4
        for (int v = lane; v < nv; v += 32) {
          const float4 f = lds_f4(base + 16u * v);
          const uint32_t u[4] = {__float_as_uint(f.x), __float_as_uint(f.y), __float_as_uint(f.z), __float_as_uint(f.w)};
          float acc = 0.f;
#pragma unroll
          for (int k = 0; k < 4; ++k) acc = fmaf(bf16lo(u[k]), bf16lo(u[k]), fmaf(bf16hi(u[k]), bf16hi(u[k]), acc));
          if (v < nva) sa += acc;
          else ss += acc;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          sa += __shfl_xor_sync(0xffffffffu, sa, o);
          ss += __shfl_xor_sync(0xffffffffu, ss, o);
        }
        if (lane == 0) ssq[r0 + r] = make_float2(sa, ss);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }
}

// w_out[n, k] = w[n, k] * beta(k), 8 bf16 per thread, grid-stride.
__global__ void __launch_bounds__(256) scale_cols_kernel(const uint4* __restrict__ w, uint4* __restrict__ w_out,
                                                         long long n_vec, int row_vecs, int wa,
                                                         const float* __restrict__ beta1,
                                                         const float* __restrict__ beta2, float s2) {
  pdl_trigger();
  pdl_wait();
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n_vec;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int k0 = static_cast<int>(i % row_vecs) * 8;
    const float* bb = k0 < wa ? beta1 + k0 : beta2 + (k0 - wa);
    const float sg = k0 < wa ? 1.f : s2;
    float4 b0 = __ldg(reinterpret_cast<const float4*>(bb)), b1 = __ldg(reinterpret_cast<const float4*>(bb + 4));
    b0 = make_float4(b0.x * sg, b0.y * sg, b0.z * sg, b0.w * sg);
    b1 = make_float4(b1.x * sg, b1.y * sg, b1.z * sg, b1.w * sg);
    const uint4 q = w[i];
    w_out[i] = make_uint4(pack_bf16(bf16lo(q.x) * b0.x, bf16hi(q.x) * b0.y), pack_bf16(bf16lo(q.y) * b0.z, bf16hi(q.y) * b0.w),
                          pack_bf16(bf16lo(q.z) * b1.x, bf16hi(q.z) * b1.y), pack_bf16(bf16lo(q.w) * b1.z, bf16hi(q.w) * b1.w));
  }
}

}  // namespace

cudaError_t launch_row_ssq(const void* z, long long rows, int w_attn, int w_ssm, float2* ssq, cudaStream_t st,
                           unsigned* status) {
  if (rows <= 0) return cudaSuccess;
  const long long row_bytes = static_cast<long long>(w_attn + w_ssm) * 2;
  if ((reinterpret_cast<uintptr_t>(z) & 15) == 0 && row_bytes % 16 == 0 && row_bytes <= SSQ_RING / 2) {
    // chunks of up to 48 KB (at most 8 rows, one per reducing warp), as many as the ring holds
    const int rpc = static_cast<int>(std::max<long long>(1, std::min<long long>(SSQ_WARPS, 49152 / row_bytes)));
    const int nst = static_cast<int>(std::min<long long>(8, SSQ_RING / (rpc * row_bytes)));
    const size_t smem = static_cast<size_t>(nst) * rpc * row_bytes + 2 * nst * 8 + 16;
    static std::atomic<uint64_t> attr_done{0};
    if (cudaError_t e = smem_attr_once(row_ssq_bulk_kernel, SSQ_RING + 2 * 8 * 8 + 16, attr_done)) return e;
    const long long nchunk = (rows + rpc - 1) / rpc;
    const unsigned grid = static_cast<unsigned>(std::min<long long>(nchunk, num_sms()));
    return launch(row_ssq_bulk_kernel, dim3(grid), dim3((SSQ_WARPS + 1) * 32), smem, st,
                  static_cast<const __nv_bfloat16*>(z), rows, w_attn, w_ssm, rpc, nst, ssq, status);
  }
  const int per_lane = ((w_attn + w_ssm) / 8 + 31) / 32;
  const unsigned grid = static_cast<unsigned>((rows + 7) / 8);
  const __nv_bfloat16* zz = static_cast<const __nv_bfloat16*>(z);
  if (per_lane <= 4) launch(row_ssq_kernel<4>, dim3(grid), dim3(256), 0, st, zz, rows, w_attn, w_ssm, ssq);
  else if (per_lane <= 8) launch(row_ssq_kernel<8>, dim3(grid), dim3(256), 0, st, zz, rows, w_attn, w_ssm, ssq);
  else if (per_lane <= 12) launch(row_ssq_kernel<12>, dim3(grid), dim3(256), 0, st, zz, rows, w_attn, w_ssm, ssq);
  else if (per_lane <= 16) launch(row_ssq_kernel<16>, dim3(grid), dim3(256), 0, st, zz, rows, w_attn, w_ssm, ssq);
  else if (per_lane <= 24) launch(row_ssq_kernel<24>, dim3(grid), dim3(256), 0, st, zz, rows, w_attn, w_ssm, ssq);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_scale_cols(const void* w, void* w_out, int N, int w_attn, int w_ssm, const float* beta1,
                              const float* beta2, cudaStream_t st, float s2) {
  const int row_vecs = (w_attn + w_ssm) / 8;
  const long long n_vec = static_cast<long long>(N) * row_vecs;
  if (n_vec <= 0) return cudaSuccess;
  const long long blocks = (n_vec + 255) / 256;
  return launch(scale_cols_kernel, dim3(static_cast<unsigned>(blocks < 4 * num_sms() ? blocks : 4 * num_sms())),
                dim3(256), 0, st, static_cast<const uint4*>(w), static_cast<uint4*>(w_out), n_vec, row_vecs, w_attn,
                beta1, beta2, s2);
}

cudaError_t launch_branch_norm(void* z, const float* beta1, const float* beta2, long long rows, int w_attn, int w_ssm,
                               float eps, bool bf16, cudaStream_t st, float s2) {
  if (rows <= 0) return cudaSuccess;
  if (bf16 && rownorm_bf16(z, z, rows, w_attn, w_ssm, beta1, beta2, eps, st, s2)) return cudaGetLastError();
  if (bf16)
    return launch(branch_norm_kernel<__nv_bfloat16>, dim3(static_cast<unsigned>(rows)), dim3(NT), 0, st,
                  static_cast<__nv_bfloat16*>(z), beta1, beta2, w_attn, w_ssm, eps, s2);
  return launch(branch_norm_kernel<float>, dim3(static_cast<unsigned>(rows)), dim3(NT), 0, st, static_cast<float*>(z),
                beta1, beta2, w_attn, w_ssm, eps, s2);
}

cudaError_t launch_rmsnorm(const void* x, void* y, long long rows, int d, float eps, bool bf16, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (bf16 && rownorm_bf16(x, y, rows, 0, d, nullptr, nullptr, eps, st)) return cudaGetLastError();
  if (bf16)
    return launch(rmsnorm_kernel<__nv_bfloat16>, dim3(static_cast<unsigned>(rows)), dim3(NT), 0, st,
                  static_cast<const __nv_bfloat16*>(x), static_cast<__nv_bfloat16*>(y), d, eps);
  return launch(rmsnorm_kernel<float>, dim3(static_cast<unsigned>(rows)), dim3(NT), 0, st,
                static_cast<const float*>(x), static_cast<float*>(y), d, eps);
}

}  // namespace hy

// ---------------------------------------------------------------------------------
// Residual stream in fp32 (stacked blocks).

namespace hy {
namespace {

// One warp per row of x [rows, d] fp32: y = gain * x / sqrt(mean(x^2) + eps) in TO (bf16 or
// fp32); with y_lo, also the bf16 rounding remainder v - float(bf16(v)) (bf16 output only).
// Two passes over the row: the second re-reads it from L1/L2.
template <typename TO>
__global__ void __launch_bounds__(256) prenorm_f32_kernel(const float* __restrict__ x, const float* __restrict__ gain,
                                                          TO* __restrict__ y, __nv_bfloat16* __restrict__ y_lo,
                                                          long long rows, int d, float eps, long long y_ld) {
  pdl_trigger();
  pdl_wait();
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float* xr = x + row * d;
  float s = 0.f;
  for (int i = lane * 8; i < d; i += 256) {
    float f[8];
    Vec8<float>::load(xr + i, f);
#pragma unroll
    for (int j = 0; j < 8; ++j) s = fmaf(f[j], f[j], s);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float r = rsqrtf(s / d + eps);
  for (int i = lane * 8; i < d; i += 256) {
    float f[8];
    Vec8<float>::load(xr + i, f);
    if (gain) {
      float g[8];
      Vec8<float>::load(gain + i, g);
#pragma unroll
      for (int j = 0; j < 8; ++j) f[j] = f[j] * r * g[j];
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) f[j] *= r;
    }
    Vec8<TO>::store(y + row * y_ld + i, f);
    if (y_lo) {
      float lo[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) lo[j] = f[j] - __bfloat162float(__float2bfloat16_rn(f[j]));
      Vec8<__nv_bfloat16>::store(y_lo + row * y_ld + i, lo);
    }
  }
}

// h[b, t, :] = float(t < M ? meta[t, :] : x[b, t - M, :]), 8 elements per thread.
__global__ void __launch_bounds__(256) prepend_f32_kernel(const __nv_bfloat16* __restrict__ x,
                                                          const __nv_bfloat16* __restrict__ meta,
                                                          float* __restrict__ h, int L, int M, int d,
                                                          long long total_vec) {
  pdl_trigger();
  pdl_wait();
  const int rv = d / 8;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total_vec;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = i / rv;
    const int e = static_cast<int>(i - row * rv) * 8;
    const long long T = L + M, b = row / T, t = row - b * T;
    const __nv_bfloat16* src = t < M ? meta + t * d + e : x + (b * L + (t - M)) * d + e;
    float f[8];
    Vec8<__nv_bfloat16>::load(src, f);
    Vec8<float>::store(h + row * d + e, f);
  }
}

// dst [cols, rows] = src [rows, cols]^T through a 32 x 32 shared tile (bf16).
__global__ void __launch_bounds__(256) transpose_bf16_kernel(const __nv_bfloat16* __restrict__ src, long long src_ld,
                                                             __nv_bfloat16* __restrict__ dst, int rows, int cols) {
  pdl_trigger();
  pdl_wait();
  __shared__ __nv_bfloat16 tile[32][33];
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 8 rows of 32 threads
  for (int k = ty; k < 32; k += 8) {
    const int r = r0 + k, c = c0 + tx;
    if (r < rows && c < cols) tile[k][tx] = src[static_cast<long long>(r) * src_ld + c];
  }
  __syncthreads();
  for (int k = ty; k < 32; k += 8) {
    const int c = c0 + k, r = r0 + tx;
    if (r < rows && c < cols) dst[static_cast<long long>(c) * rows + r] = tile[tx][k];
  }
}

// dst + b * stride = src (16-byte units), grid-stride over batch x units.
__global__ void __launch_bounds__(256) broadcast_kernel(const uint4* __restrict__ src, long long units,
                                                        uint8_t* __restrict__ dst, long long stride, int batch) {
  pdl_trigger();
  pdl_wait();
  const long long total = units * batch;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long b = i / units, u = i - b * units;
    reinterpret_cast<uint4*>(dst + b * stride)[u] = src[u];
  }
}

}  // namespace

cudaError_t launch_broadcast(const void* src, size_t bytes, void* dst, size_t dst_stride, int batch,
                             cudaStream_t st) {
  if (bytes == 0 || batch <= 0) return cudaSuccess;
  if (bytes % 16 || dst_stride % 16 || (reinterpret_cast<uintptr_t>(src) & 15) || (reinterpret_cast<uintptr_t>(dst) & 15))
    return cudaErrorInvalidValue;
  const long long units = static_cast<long long>(bytes / 16), total = units * batch;
  const long long blocks = (total + 255) / 256;
  return launch(broadcast_kernel, dim3(static_cast<unsigned>(blocks < 4 * num_sms() ? blocks : 4 * num_sms())),
                dim3(256), 0, st, static_cast<const uint4*>(src), units, static_cast<uint8_t*>(dst),
                static_cast<long long>(dst_stride), batch);
}

cudaError_t launch_prenorm_f32(const float* x, const float* gain, void* y, void* y_lo, long long rows, int d,
                               float eps, cudaStream_t st, long long y_ld) {
  if (rows <= 0) return cudaSuccess;
  if (d % 8 || (y_ld && (y_ld < d || y_ld % 8))) return cudaErrorInvalidValue;
  const unsigned grid = static_cast<unsigned>((rows + 7) / 8);
  return launch(prenorm_f32_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, x, gain,
                static_cast<__nv_bfloat16*>(y), static_cast<__nv_bfloat16*>(y_lo), rows, d, eps, y_ld ? y_ld : d);
}

namespace {
__global__ void __launch_bounds__(256) split_hi_lo_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ hi,
                                                          __nv_bfloat16* __restrict__ lohi, int rows, int cols) {
  pdl_trigger();
  pdl_wait();
  const long long n = static_cast<long long>(rows) * cols;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / cols, c = i - r * cols;
    const float v = src[i];
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    hi[i] = h;
    lohi[r * 2 * cols + c] = __float2bfloat16_rn(v - __bfloat162float(h));
    lohi[r * 2 * cols + cols + c] = h;
  }
}
}  // namespace

cudaError_t launch_split_hi_lo(const float* src, void* hi, void* lohi, int rows, int cols, cudaStream_t st) {
  const long long n = static_cast<long long>(rows) * cols;
  if (n <= 0) return cudaSuccess;
  const long long blocks = (n + 255) / 256;
  return launch(split_hi_lo_kernel, dim3(static_cast<unsigned>(blocks < 4 * num_sms() ? blocks : 4 * num_sms())),
                dim3(256), 0, st, src, static_cast<__nv_bfloat16*>(hi), static_cast<__nv_bfloat16*>(lohi), rows, cols);
}

cudaError_t launch_prenorm_f32_out_f32(const float* x, const float* gain, float* y, long long rows, int d, float eps,
                                       cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (d % 8) return cudaErrorInvalidValue;
  const unsigned grid = static_cast<unsigned>((rows + 7) / 8);
  return launch(prenorm_f32_kernel<float>, dim3(grid), dim3(256), 0, st, x, gain, y,
                static_cast<__nv_bfloat16*>(nullptr), rows, d, eps, static_cast<long long>(d));
}

cudaError_t launch_prepend_f32(const void* x, const void* meta, float* h, int batch, int L, int M, int d,
                               cudaStream_t st) {
  const long long total = static_cast<long long>(batch) * (L + M) * (d / 8);
  if (total <= 0) return cudaSuccess;
  if (d % 8) return cudaErrorInvalidValue;
  const long long blocks = (total + 255) / 256;
  return launch(prepend_f32_kernel, dim3(static_cast<unsigned>(blocks < 8 * num_sms() ? blocks : 8 * num_sms())),
                dim3(256), 0, st, static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(meta), h, L,
                M, d, total);
}

cudaError_t launch_transpose_bf16(const void* src, long long src_ld, void* dst, int rows, int cols, cudaStream_t st) {
  if (rows <= 0 || cols <= 0) return cudaSuccess;
  dim3 grid((cols + 31) / 32, (rows + 31) / 32);
  return launch(transpose_bf16_kernel, grid, dim3(256), 0, st, static_cast<const __nv_bfloat16*>(src), src_ld,
                static_cast<__nv_bfloat16*>(dst), rows, cols);
}

}  // namespace hy
