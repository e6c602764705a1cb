// gemv.cu -- products with a handful of rows (the generation step: one row per sequence)
// on the CUDA cores, C = A W^T for A [M <= 8, K] and W [N, K] bf16, with the same column-
// segment epilogues as the tensor-core GEMM (store, SiLU, softplus(. + bias); bf16 or fp32
// output at a segment's own pointer and row stride).
//
// A 128-row tensor-core tile would spend 120 of its rows on nothing and, with N / 256
// tiles, leave most SMs idle (out_proj of a 2048-wide model: 8 CTAs); here the product is
// a stream over W, which sets its time: every W row is read once, 16 bytes per lane per
// load, by a warp that owns two rows; A is staged once per CTA in shared memory.  fp32
// accumulation; the warp's partial sums are combined by shuffles.
#include "hy_common.cuh"
#include "hy_kernels.h"

namespace hy {
namespace {

constexpr int GV_WARPS = 8;   // warps per CTA
constexpr int GV_ROWS = 2;    // W rows per warp
constexpr int GV_MAX_M = 8;

struct GemvParams {
  const __nv_bfloat16* a;
  const __nv_bfloat16* w;
  int M, K, N, nseg;
  Seg seg[kMaxSegs];
};

// Eight bf16 values (one 16-byte vector) as fp32.
__device__ __forceinline__ void bf16x8(const uint4 v, float (&f)[8]) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(u[i] << 16);
    f[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <int M>
__global__ void __launch_bounds__(GV_WARPS * 32) gemv_bf16_kernel(const __grid_constant__ GemvParams p) {
  extern __shared__ uint4 sa[];  // A: [M][K / 8] 16-byte vectors
  pdl_trigger();
  const int kv = p.K / 8;
  pdl_wait();
  for (int i = threadIdx.x; i < M * kv; i += blockDim.x) sa[i] = reinterpret_cast<const uint4*>(p.a)[i];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = (blockIdx.x * GV_WARPS + warp) * GV_ROWS;
  if (n0 >= p.N) return;
  float acc[GV_ROWS][M];
#pragma unroll
  for (int r = 0; r < GV_ROWS; ++r)
#pragma unroll
    for (int m = 0; m < M; ++m) acc[r][m] = 0.f;
  const uint4* wr[GV_ROWS];
#pragma unroll
  for (int r = 0; r < GV_ROWS; ++r)
    wr[r] = reinterpret_cast<const uint4*>(p.w) + static_cast<long long>(min(n0 + r, p.N - 1)) * kv;
#pragma unroll 4
  for (int k = lane; k < kv; k += 32) {
    float wf[GV_ROWS][8];
#pragma unroll
    for (int r = 0; r < GV_ROWS; ++r) bf16x8(ldg_stream(wr[r] + k), wf[r]);
#pragma unroll
    for (int m = 0; m < M; ++m) {
      float xf[8];
      bf16x8(sa[m * kv + k], xf);
#pragma unroll
      for (int r = 0; r < GV_ROWS; ++r)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[r][m] = fmaf(wf[r][e], xf[e], acc[r][m]);
    }
  }
#pragma unroll
  for (int r = 0; r < GV_ROWS; ++r)
#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[r][m] += __shfl_xor_sync(0xffffffffu, acc[r][m], o);
  // lane r * M + m stores output (m, n0 + r)
#pragma unroll
  for (int r = 0; r < GV_ROWS; ++r) {
#pragma unroll
    for (int m = 0; m < M; ++m) {
      if (lane != r * M + m) continue;
      const int n = n0 + r;
      if (n >= p.N) continue;
      int s = 0;
      while (s + 1 < p.nseg && n >= p.seg[s].col1) ++s;
      const Seg& sg = p.seg[s];
      if (n < sg.col0 || n >= sg.col1) continue;
      float v = acc[r][m];
      if (sg.op == SEG_SILU) v = silu_f(v);
      else if (sg.op == SEG_SOFTPLUS_BIAS) v = softplus_f(v + sg.bias[n - sg.col0]);
      const long long off = static_cast<long long>(m) * sg.ld + (n - sg.col0);
      if (sg.out_f32) static_cast<float*>(sg.ptr)[off] = v;
      else static_cast<__nv_bfloat16*>(sg.ptr)[off] = __float2bfloat16_rn(v);
    }
  }
}

// The same product split along K, for long rows (K >= 2048) whose W rows alone would not
// fill the GPU (N / 16 row pairs short of two CTAs per SM): a CTA owns two W rows, its 256 threads
// take every 256th 16-byte vector of K (A read straight from L2), and the partial sums
// meet in shared memory.
template <int M>
__global__ void __launch_bounds__(256) gemv_bf16_splitk_kernel(const __grid_constant__ GemvParams p) {
  __shared__ float red[GV_WARPS][GV_ROWS][M];
  pdl_trigger();
  pdl_wait();
  const int kv = p.K / 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * GV_ROWS;
  float acc[GV_ROWS][M];
#pragma unroll
  for (int r = 0; r < GV_ROWS; ++r)
#pragma unroll
    for (int m = 0; m < M; ++m) acc[r][m] = 0.f;
  const uint4* wr[GV_ROWS];
#pragma unroll
  for (int r = 0; r < GV_ROWS; ++r)
    wr[r] = reinterpret_cast<const uint4*>(p.w) + static_cast<long long>(min(n0 + r, p.N - 1)) * kv;
  const uint4* a4 = reinterpret_cast<const uint4*>(p.a);
#pragma unroll 4
  for (int k = threadIdx.x; k < kv; k += 256) {
    float wf[GV_ROWS][8];
#pragma unroll
    for (int r = 0; r < GV_ROWS; ++r) bf16x8(ldg_stream(wr[r] + k), wf[r]);
#pragma unroll
    for (int m = 0; m < M; ++m) {
      float xf[8];
      bf16x8(a4[m * kv + k], xf);
#pragma unroll
      for (int r = 0; r < GV_ROWS; ++r)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[r][m] = fmaf(wf[r][e], xf[e], acc[r][m]);
    }
  }
#pragma unroll
  for (int r = 0; r < GV_ROWS; ++r)
#pragma unroll
    for (int m = 0; m < M; ++m) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[r][m] += __shfl_xor_sync(0xffffffffu, acc[r][m], o);
      if (lane == 0) red[warp][r][m] = acc[r][m];
    }
  __syncthreads();
  if (threadIdx.x < GV_ROWS * M) {
    const int r = threadIdx.x / M, m = threadIdx.x % M, n = n0 + r;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < GV_WARPS; ++w) v += red[w][r][m];
    if (n < p.N) {
      int s = 0;
      while (s + 1 < p.nseg && n >= p.seg[s].col1) ++s;
      const Seg& sg = p.seg[s];
      if (n >= sg.col0 && n < sg.col1) {
        if (sg.op == SEG_SILU) v = silu_f(v);
        else if (sg.op == SEG_SOFTPLUS_BIAS) v = softplus_f(v + sg.bias[n - sg.col0]);
        const long long off = static_cast<long long>(m) * sg.ld + (n - sg.col0);
        if (sg.out_f32) static_cast<float*>(sg.ptr)[off] = v;
        else static_cast<__nv_bfloat16*>(sg.ptr)[off] = __float2bfloat16_rn(v);
      }
    }
  }
}

template <int M>
cudaError_t launch_m(const GemvParams& p, cudaStream_t st) {
  const int cols = GV_WARPS * GV_ROWS;
  if ((p.N + cols - 1) / cols < 2 * num_sms() && p.K >= 2048)
    return launch(gemv_bf16_splitk_kernel<M>, dim3((p.N + GV_ROWS - 1) / GV_ROWS), dim3(256), 0, st, p);
  const size_t smem = static_cast<size_t>(M) * p.K * 2;
  static std::atomic<uint64_t> attr_done{0};   // the attribute is set once, to the largest A accepted
  if (cudaError_t e = smem_attr_once(gemv_bf16_kernel<M>, 96 * 1024, attr_done)) return e;
  return launch(gemv_bf16_kernel<M>, dim3((p.N + cols - 1) / cols), dim3(GV_WARPS * 32), smem, st, p);
}

}  // namespace

// Whether gemv_bf16 takes this product: plain A with rows back to back, at most 8 rows,
// the segment epilogue, K a multiple of 8 (16-byte vectors), A staged in at most 96 KB.
bool gemv_bf16_takes(const GemmDesc& g) {
  return !g.meta_mode && g.a_rows >= 1 && g.a_rows <= GV_MAX_M && (g.a_ld == 0 || g.a_ld == g.K) &&
         g.epi == EPI_SEGMENTS && g.K2 == 0 && g.remap_L == 0 && g.dual_k_blocks == 0 && g.K % 8 == 0 &&
         g.a_rows * g.K * 2 <= 96 * 1024 && (reinterpret_cast<uintptr_t>(g.a) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(g.w) & 15) == 0 && g.nseg >= 1 && g.nseg <= kMaxSegs;
}

cudaError_t launch_gemv_bf16(const GemmDesc& g, cudaStream_t st) {
  if (!gemv_bf16_takes(g)) return cudaErrorInvalidValue;
  GemvParams p{};
  p.a = static_cast<const __nv_bfloat16*>(g.a);
  p.w = static_cast<const __nv_bfloat16*>(g.w);
  p.M = static_cast<int>(g.a_rows);
  p.K = g.K;
  p.N = g.N;
  p.nseg = g.nseg;
  for (int i = 0; i < g.nseg; ++i) p.seg[i] = g.seg[i];
  switch (p.M) {
    case 1: return launch_m<1>(p, st);
    case 2: return launch_m<2>(p, st);
    case 3: return launch_m<3>(p, st);
    case 4: return launch_m<4>(p, st);
    case 5: return launch_m<5>(p, st);
    case 6: return launch_m<6>(p, st);
    case 7: return launch_m<7>(p, st);
    default: return launch_m<8>(p, st);
  }
}

}  // namespace hy
