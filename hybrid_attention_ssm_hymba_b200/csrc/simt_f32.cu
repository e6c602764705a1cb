// simt_f32.cu -- the fp32 path (CUDA cores, fp32 arithmetic, no tensor cores; TF32
// would not meet a 1e-4 tolerance): a tiled SIMT GEMM with the same epilogues as
// the tensor-core GEMM, and a warp-per-query attention.  It serves layers whose
// cfg.dtype is HYMBA_F32, e.g. the tiny fp32 hybrid-head layer.
#include "hy_common.cuh"
#include "hy_kernels.h"

namespace hy {
namespace {

constexpr int TB = 64, TK = 16;

struct F32GemmParams {
  int meta_mode;
  const float* a;  // plain A [rows, K]
  const float* x;  // meta mode: x [B, L, K], meta [M, K]
  const float* meta;
  int L, n_meta, T;
  long long rows;  // output rows
  const float* w;  // [N, K]
  int N, K;
  int epi;
  int nseg;
  Seg seg[kMaxSegs];
  const float* resid;
  long long resid_ld;
  float* out;
  long long out_ld;
  int swiglu_F;
  int remap_L, remap_T, remap_M;   // segment rows: r -> (r / L) T + M + r % L when remap_L > 0
};

__device__ __forceinline__ const float* a_row(const F32GemmParams& p, long long r) {
  if (!p.meta_mode) return p.a + r * p.K;
  const long long b = r / p.T;
  const int t = static_cast<int>(r - b * p.T);
  if (t < p.n_meta) return p.meta + static_cast<long long>(t) * p.K;
  return p.x + (b * p.L + (t - p.n_meta)) * p.K;
}

__device__ __forceinline__ void store_elem(const F32GemmParams& p, long long row, int col, float v) {
  int s = 0;
  while (s + 1 < p.nseg && col >= p.seg[s].col1) ++s;
  const Seg& sg = p.seg[s];
  if (col < sg.col0 || col >= sg.col1) return;
  if (sg.op == SEG_SILU) v = v / (1.f + expf(-v));
  else if (sg.op == SEG_SOFTPLUS_BIAS) {
    const float z = v + sg.bias[col - sg.col0];
    v = z > 20.f ? z : log1pf(expf(z));
  }
  static_cast<float*>(sg.ptr)[row * sg.ld + (col - sg.col0)] = v;
}

// C tile 64 x 64, 256 threads x (4 x 4); SWIGLU computes gate and up tiles together.
template <bool SWIGLU>
__global__ void __launch_bounds__(256) gemm_f32_kernel(const __grid_constant__ F32GemmParams p) {
  pdl_trigger();
  pdl_wait();
  __shared__ float As[TK][TB + 1];
  __shared__ float Ws[TK][TB + 1];
  __shared__ float Us[SWIGLU ? TK : 1][TB + 1];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const long long m0 = static_cast<long long>(blockIdx.y) * TB;
  const int n0 = blockIdx.x * TB;
  float acc[4][4] = {}, accu[4][4] = {};
  for (int k0 = 0; k0 < p.K; k0 += TK) {
    for (int e = threadIdx.x; e < TB * TK; e += 256) {
      const int r = e / TK, k = e % TK;
      const long long gr = m0 + r;
      const int gk = k0 + k;
      As[k][r] = (gr < p.rows && gk < p.K) ? a_row(p, gr)[gk] : 0.f;
      const int gn = n0 + r;
      const int wn = SWIGLU ? gn : gn;
      Ws[k][r] = (wn < (SWIGLU ? p.swiglu_F : p.N) && gk < p.K) ? p.w[static_cast<long long>(wn) * p.K + gk] : 0.f;
      if (SWIGLU)
        Us[k][r] = (gn < p.swiglu_F && gk < p.K) ? p.w[static_cast<long long>(p.swiglu_F + gn) * p.K + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < TK; ++k) {
      float av[4], wv[4], uv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        av[i] = As[k][ty * 4 + i];
        wv[i] = Ws[k][tx * 4 + i];
        if (SWIGLU) uv[i] = Us[k][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(av[i], wv[j], acc[i][j]);
          if (SWIGLU) accu[i][j] = fmaf(av[i], uv[j], accu[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long row = m0 + ty * 4 + i;
    if (row >= p.rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = n0 + tx * 4 + j;
      if (SWIGLU) {
        if (col < p.swiglu_F) {
          const float g = acc[i][j];
          p.out[row * p.out_ld + col] = g / (1.f + expf(-g)) * accu[i][j];
        }
      } else if (col < p.N) {
        if (p.epi == EPI_RESIDUAL)
          p.out[row * p.out_ld + col] = p.resid[row * p.resid_ld + col] + acc[i][j];
        else
          store_elem(p, p.remap_L ? (row / p.remap_L) * p.remap_T + p.remap_M + row % p.remap_L : row, col,
                     acc[i][j]);
      }
    }
  }
}

// One warp per (sequence, query head, query row); fp32 online softmax over the
// visible keys: j <= i and (window < 0 or i - j <= window or j < n_meta).
__global__ void __launch_bounds__(128) attention_f32_kernel(const float* __restrict__ q, long long q_ld,
                                                            const float* __restrict__ k,
                                                            const float* __restrict__ v, long long kv_ld,
                                                            float* __restrict__ out, long long out_ld, int T, int Hq,
                                                            int Hkv, int dh, int n_meta, int window, int batch,
                                                            long long kv_rows) {
  pdl_trigger();
  pdl_wait();
  const long long wid = static_cast<long long>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long total = static_cast<long long>(batch) * Hq * T;
  if (wid >= total) return;
  const int i = static_cast<int>(wid % T);
  const int h = static_cast<int>((wid / T) % Hq);
  const int b = static_cast<int>(wid / (static_cast<long long>(T) * Hq));
  const int kvh = h / (Hq / Hkv);
  const float scale = rsqrtf(static_cast<float>(dh));
  const long long qrow = static_cast<long long>(b) * T + i;
  float qv[4], acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int d = lane + 32 * e;
    qv[e] = d < dh ? q[qrow * q_ld + h * dh + d] : 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int j = 0; j <= i; ++j) {
    if (!(window < 0 || i - j <= window || j < n_meta)) continue;
    const long long krow = static_cast<long long>(b) * kv_rows + j;
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int d = lane + 32 * e;
      if (d < dh) s = fmaf(qv[e], k[krow * kv_ld + kvh * dh + d], s);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    s *= scale;
    const float mn = fmaxf(m, s);
    const float corr = expf(m - mn), pj = expf(s - mn);
    l = l * corr + pj;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int d = lane + 32 * e;
      const float vv = d < dh ? v[krow * kv_ld + kvh * dh + d] : 0.f;
      acc[e] = acc[e] * corr + pj * vv;
    }
    m = mn;
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int d = lane + 32 * e;
    if (d < dh) out[qrow * out_ld + h * dh + d] = acc[e] / l;
  }
}

}  // namespace

cudaError_t launch_gemm_f32(const GemmDesc& g, cudaStream_t st) {
  F32GemmParams p{};
  p.meta_mode = g.meta_mode ? 1 : 0;
  p.a = static_cast<const float*>(g.a);
  p.x = static_cast<const float*>(g.x);
  p.meta = static_cast<const float*>(g.meta);
  p.L = g.L;
  p.n_meta = g.n_meta;
  p.T = g.L + g.n_meta;
  p.rows = g.meta_mode ? static_cast<long long>(g.batch) * p.T : g.a_rows;
  p.w = static_cast<const float*>(g.w);
  p.N = g.N;
  p.K = g.K;
  p.epi = g.epi;
  p.nseg = g.nseg;
  for (int i = 0; i < g.nseg; ++i) p.seg[i] = g.seg[i];
  p.resid = static_cast<const float*>(g.resid);
  p.resid_ld = g.resid_ld;
  p.out = static_cast<float*>(g.out);
  p.out_ld = g.out_ld;
  p.swiglu_F = g.swiglu_F;
  p.remap_L = g.remap_L;
  p.remap_T = g.remap_T;
  p.remap_M = g.remap_M;
  if (p.rows <= 0) return cudaSuccess;
  const int ncols = g.epi == EPI_SWIGLU ? g.swiglu_F : g.N;
  dim3 grid((ncols + TB - 1) / TB, static_cast<unsigned>((p.rows + TB - 1) / TB));
  if (g.epi == EPI_SWIGLU) return launch(gemm_f32_kernel<true>, grid, dim3(256), 0, st, p);
  return launch(gemm_f32_kernel<false>, grid, dim3(256), 0, st, p);
}

cudaError_t launch_attention_f32(const AttnDesc& a, cudaStream_t st) {
  const long long total = static_cast<long long>(a.batch) * a.n_q_heads * a.T;
  if (total <= 0) return cudaSuccess;
  return launch(attention_f32_kernel, dim3(static_cast<unsigned>((total + 3) / 4)), dim3(128), 0, st,
                static_cast<const float*>(a.q), a.q_ld, static_cast<const float*>(a.k),
                static_cast<const float*>(a.v), a.kv_ld, static_cast<float*>(a.out), a.out_ld, a.T, a.n_q_heads,
                a.n_kv_heads, a.head_dim, a.n_meta, a.window, a.batch, a.kv_rows > 0 ? a.kv_rows : a.T);
}

}  // namespace hy
