// adaLN-single time conditioning on sm_100a: the paper §2.1 "Time conditioning" of
// "Nemotron-TwoTower: Diffusion Language Modeling with Pretrained AR Context" (adaLN-single as in
// PixArt-alpha: one global MLP from the diffusion time to shared shift/scale/gate, plus a learned
// per-layer embedding).
//
//   COND             tau -> mod[B][3][D]   two launches: per sequence the sinusoid and the two
//                                          W-wide layers; then the W->3D layer tiled over 32-row
//                                          slices of W3, each read once for the whole batch
//   NORM_MODULATE    RMSNorm prologue modulated by (shift, scale): one CTA per token row
//   GATED_RESIDUAL   h + gate * f: a vectorised elementwise pass
// All arithmetic is fp32 (the timestep sinusoid in fp64); bf16 tensors are widened on load and
// rounded to nearest on store.
#include <algorithm>
#include <cmath>

#include "tt_common.cuh"
#include "tt_internal.h"

namespace tt {

constexpr int kAdalnThreads = 256;

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + expf(-x)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// phi(tau) = [cos(1000 tau w_k), sin(1000 tau w_k)], w_k = 10000^(-k/(F/2)). The angle (up to
// 1000 rad) is formed and reduced modulo 2 pi in double, so the single-precision sincos only sees
// |angle| <= pi.
__device__ __forceinline__ void phi_row(float tau, int F, float* dst, int tid, int nthreads) {
  const int half = F / 2;
  const double t = 1000.0 * (double)tau;
  const double two_pi = 6.283185307179586476925286766559;
  for (int k = tid; k < half; k += nthreads) {
    const double w = exp(-9.2103403719761836 * (double)k / (double)half);   // ln(10000) = 9.2103...
    double a = t * w;
    a -= two_pi * rint(a * (1.0 / two_pi));
    float sv, cv;
    sincosf((float)a, &sv, &cv);
    dst[k] = cv;
    dst[half + k] = sv;
  }
}

constexpr int kMaxWidth = 1024;   // F and W bound (host-validated)

// y[o] = act(W[o, :] . x + bias[o]) for o < OUT, x in shared memory; each warp takes four rows at
// a time (four independent dot products and reductions in flight), lanes stride the row in float4.
template <bool kSilu>
__device__ __forceinline__ void cta_gemv(const float* __restrict__ Wt, const float* __restrict__ bias,
                                         const float* x, int IN, int OUT, float* y) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int o0 = warp * 4; o0 < OUT; o0 += nwarps * 4) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int i = lane * 4; i < IN; i += 128) {
      const float4 xv = *reinterpret_cast<const float4*>(x + i);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        if (o0 + r < OUT) {
          const float4 wv = *reinterpret_cast<const float4*>(Wt + (size_t)(o0 + r) * IN + i);
          acc[r] = fmaf(wv.x, xv.x, fmaf(wv.y, xv.y, fmaf(wv.z, xv.z, fmaf(wv.w, xv.w, acc[r]))));
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[r] = warp_sum(acc[r]);
    if (lane < 4 && o0 + lane < OUT) {
      const float v = (lane == 0 ? acc[0] : lane == 1 ? acc[1] : lane == 2 ? acc[2] : acc[3]) + bias[o0 + lane];
      y[o0 + lane] = kSilu ? silu_f(v) : v;
    }
  }
}

// COND, first launch: one CTA per sequence b computes a2[b] = SiLU(W2 SiLU(W1 phi(tau_b) + b1) + b2).
__global__ void __launch_bounds__(kAdalnThreads) adaln_hidden_kernel(const float* __restrict__ tau,
                                                                     const float* __restrict__ w1,
                                                                     const float* __restrict__ b1,
                                                                     const float* __restrict__ w2,
                                                                     const float* __restrict__ b2, int F, int W,
                                                                     float* __restrict__ a2,
                                                                     const int32_t* skip_if) {
  __shared__ __align__(16) float s_phi[kMaxWidth];
  __shared__ __align__(16) float s_a1[kMaxWidth];
  pdl_trigger();
  pdl_wait();
  if (skip_requested(skip_if)) return;
  const int b = blockIdx.x;
  phi_row(tau[b], F, s_phi, threadIdx.x, blockDim.x);
  __syncthreads();
  cta_gemv<true>(w1, b1, s_phi, F, W, s_a1);
  __syncthreads();
  cta_gemv<true>(w2, b2, s_a1, W, W, a2 + (size_t)b * W);
}

// COND, second launch: mod[b][o] = W3[o, :] . a2[b] + b3[o] + layer_emb[o] for o < 3D. A CTA
// owns 32 rows of W3 (in shared memory, rows padded by 4 floats so that the quarter-warp float4
// reads of 8 rows hit distinct banks) and every sequence: lane = row, warp = a group of sequences
// whose a2 rows are read as broadcasts; chunks of up to 64 sequences at a time (fewer for wide W,
// so that the chunk and the W3 slice fit in shared memory).
constexpr int kOutRows = 32;
constexpr int kOutSeqChunk = 64;
inline int out_seq_chunk(int W) { return W <= 256 ? 64 : (W <= 512 ? 32 : 16); }
inline size_t out_smem_bytes(int W) {
  return sizeof(float) * ((size_t)kOutRows * (W + 4) + (size_t)out_seq_chunk(W) * W);
}

__global__ void __launch_bounds__(kAdalnThreads) adaln_out_kernel(const float* __restrict__ w3,
                                                                  const float* __restrict__ b3,
                                                                  const float* __restrict__ emb,
                                                                  const float* __restrict__ a2, int B, int W,
                                                                  int OUT, int chunk, float* __restrict__ mod,
                                                                  const int32_t* skip_if) {
  extern __shared__ __align__(16) float s_dyn[];
  const int WP = W + 4;
  float* s_w = s_dyn;                          // [32][W + 4]
  float* s_a = s_dyn + kOutRows * WP;          // [chunk][W]
  pdl_trigger();
  pdl_wait();
  if (skip_requested(skip_if)) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int o0 = blockIdx.x * kOutRows;
  const int nrow = min(kOutRows, OUT - o0);
  const int wv = W / 4;
  for (int i = threadIdx.x; i < kOutRows * wv; i += blockDim.x) {
    const int r = i / wv, c = i - r * wv;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < nrow) v = reinterpret_cast<const float4*>(w3 + (size_t)(o0 + r) * W)[c];
    *reinterpret_cast<float4*>(s_w + r * WP + 4 * c) = v;
  }
  const int o = o0 + lane;
  const float add = (lane < nrow) ? b3[o] + emb[o] : 0.f;
  for (int c0 = 0; c0 < B; c0 += chunk) {
    const int nb = min(chunk, B - c0);
    __syncthreads();   // the previous chunk is consumed (and, the first time, s_w is written)
    for (int i = threadIdx.x; i < nb * wv; i += blockDim.x)
      reinterpret_cast<float4*>(s_a)[i] = reinterpret_cast<const float4*>(a2 + (size_t)c0 * W)[i];
    __syncthreads();
    float acc[kOutSeqChunk / 8];
#pragma unroll
    for (int i = 0; i < kOutSeqChunk / 8; ++i) acc[i] = 0.f;
    for (int k = 0; k < W; k += 4) {
      const float4 w = *reinterpret_cast<const float4*>(s_w + lane * WP + k);
#pragma unroll
      for (int i = 0; i < kOutSeqChunk / 8; ++i) {
        const int bb = warp + 8 * i;
        if (bb < nb) {
          const float4 x = *reinterpret_cast<const float4*>(s_a + bb * W + k);
          acc[i] = fmaf(w.x, x.x, fmaf(w.y, x.y, fmaf(w.z, x.z, fmaf(w.w, x.w, acc[i]))));
        }
      }
    }
    if (lane < nrow) {
#pragma unroll
      for (int i = 0; i < kOutSeqChunk / 8; ++i) {
        const int bb = warp + 8 * i;
        if (bb < nb) mod[(size_t)(c0 + bb) * OUT + o] = acc[i] + add;
      }
    }
  }
}

template <typename T>
struct Io;
template <>
struct Io<float> {
  static constexpr int kN = 4;
  __device__ static void load(const void* p, size_t i, float* x) {
    const float4 v = reinterpret_cast<const float4*>(p)[i];
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  }
  __device__ static void store(void* p, size_t i, const float* x) {
    reinterpret_cast<float4*>(p)[i] = make_float4(x[0], x[1], x[2], x[3]);
  }
};
template <>
struct Io<__nv_bfloat16> {
  static constexpr int kN = 8;
  __device__ static void load(const void* p, size_t i, float* x) {
    const uint4 v = reinterpret_cast<const uint4*>(p)[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x[2 * k] = __uint_as_float(w[k] << 16);
      x[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  }
  __device__ static void store(void* p, size_t i, const float* x) {
    uint4 v;
    v.x = pack_bf16x2(x[0], x[1]);
    v.y = pack_bf16x2(x[2], x[3]);
    v.z = pack_bf16x2(x[4], x[5]);
    v.w = pack_bf16x2(x[6], x[7]);
    reinterpret_cast<uint4*>(p)[i] = v;
  }
};

// One CTA per token row (b, s): y = h / sqrt(mean(h^2) + eps) * w * (1 + scale_b) + shift_b.
template <typename T>
__global__ void __launch_bounds__(kAdalnThreads) adaln_norm_modulate_kernel(const void* __restrict__ h,
                                                                            const float* __restrict__ norm_w,
                                                                            const float* __restrict__ mod,
                                                                            int S, int D, float eps,
                                                                            void* __restrict__ out,
                                                                            const int32_t* skip_if) {
  constexpr int N = Io<T>::kN;
  pdl_trigger();
  pdl_wait();
  if (skip_requested(skip_if)) return;
  const int row = blockIdx.x;
  const int b = row / S;
  const int nv = D / N;
  const size_t vbase = (size_t)row * nv;
  const float* shift = mod + (size_t)b * 3 * D;
  const float* scale = shift + D;
  float ss = 0.f;
  for (int v = threadIdx.x; v < nv; v += blockDim.x) {
    float x[N];
    Io<T>::load(h, vbase + v, x);
#pragma unroll
    for (int k = 0; k < N; ++k) ss = fmaf(x[k], x[k], ss);
  }
  __shared__ float s_part[kAdalnThreads / 32];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += s_part[w];
  const float r = 1.0f / sqrtf(tot / (float)D + eps);
  for (int v = threadIdx.x; v < nv; v += blockDim.x) {
    float x[N];
    Io<T>::load(h, vbase + v, x);
    const int j0 = v * N;
#pragma unroll
    for (int k = 0; k < N; ++k) {
      const int j = j0 + k;
      x[k] = fmaf(x[k] * r * norm_w[j], 1.0f + scale[j], shift[j]);
    }
    Io<T>::store(out, vbase + v, x);
  }
}

// out = h + gate_b * f, elementwise over [B][S][D].
template <typename T>
__global__ void __launch_bounds__(kAdalnThreads) adaln_gated_residual_kernel(const void* __restrict__ h,
                                                                             const void* __restrict__ f,
                                                                             const float* __restrict__ mod,
                                                                             int S, int D, size_t nvec,
                                                                             void* out, const int32_t* skip_if) {
  constexpr int N = Io<T>::kN;
  pdl_trigger();
  pdl_wait();
  if (skip_requested(skip_if)) return;
  const int nv_row = D / N;
  for (size_t v = blockIdx.x * (size_t)blockDim.x + threadIdx.x; v < nvec; v += (size_t)gridDim.x * blockDim.x) {
    const size_t row = v / nv_row;
    const int j0 = (int)(v - row * nv_row) * N;
    const int b = (int)(row / S);
    const float* gate = mod + (size_t)b * 3 * D + 2 * D;
    float x[N], y[N];
    Io<T>::load(h, v, x);
    Io<T>::load(f, v, y);
#pragma unroll
    for (int k = 0; k < N; ++k) x[k] = fmaf(gate[j0 + k], y[k], x[k]);
    Io<T>::store(out, v, x);
  }
}

size_t adaln_workspace_bytes(const tt_adaln_args_t* a) {
  if (a->op == TT_ADALN_COND) return kHeaderBytes + sizeof(float) * (size_t)a->batch * a->mlp_width;
  return kHeaderBytes;
}

int adaln_launch(const tt_adaln_args_t* a, void* ws, cudaStream_t stream) {
  const int B = a->batch, D = a->hidden;
  if (a->op == TT_ADALN_COND) {
    float* a2 = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kHeaderBytes);
    const int F = a->freq_dim, W = a->mlp_width, OUT = 3 * D;
    launch_pdl(adaln_hidden_kernel, dim3(B), dim3(kAdalnThreads), 0, stream, a->tau, a->w1, a->b1, a->w2, a->b2, F,
               W, a2, a->skip_if);
    const size_t smem = out_smem_bytes(W);
    static unsigned long long attr_done = 0;   // bit per device ordinal (< 64): the opt-in for W up to 1024
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return TT_ERR_CUDA;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(__atomic_load_n(&attr_done, __ATOMIC_ACQUIRE) & bit)) {
      size_t max_smem = 0;
      for (int w = 256; w <= kMaxWidth; w *= 2) max_smem = std::max(max_smem, out_smem_bytes(w));
      if (cudaFuncSetAttribute(adaln_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)max_smem) !=
          cudaSuccess)
        return TT_ERR_CUDA;
      __atomic_fetch_or(&attr_done, bit, __ATOMIC_ACQ_REL);
    }
    launch_pdl(adaln_out_kernel, dim3((OUT + kOutRows - 1) / kOutRows), dim3(kAdalnThreads), smem, stream, a->w3,
               a->b3, a->layer_emb, a2, B, W, OUT, out_seq_chunk(W), a->mod, a->skip_if);
  } else if (a->op == TT_ADALN_NORM_MODULATE) {
    const int rows = B * a->block_size;
    if (a->dtype == TT_BF16)
      launch_pdl(adaln_norm_modulate_kernel<__nv_bfloat16>, dim3(rows), dim3(kAdalnThreads), 0, stream, a->h,
                 a->norm_w, (const float*)a->mod, a->block_size, D, a->eps, a->out, a->skip_if);
    else
      launch_pdl(adaln_norm_modulate_kernel<float>, dim3(rows), dim3(kAdalnThreads), 0, stream, a->h, a->norm_w,
                 (const float*)a->mod, a->block_size, D, a->eps, a->out, a->skip_if);
  } else {
    const int N = (a->dtype == TT_BF16) ? 8 : 4;
    const size_t nvec = (size_t)B * a->block_size * D / N;
    const int sms = device_sm_count();
    size_t grid = (nvec + kAdalnThreads - 1) / kAdalnThreads;
    grid = grid < (size_t)sms * 8 ? grid : (size_t)sms * 8;
    if (grid == 0) grid = 1;
    if (a->dtype == TT_BF16)
      launch_pdl(adaln_gated_residual_kernel<__nv_bfloat16>, dim3((unsigned)grid), dim3(kAdalnThreads), 0, stream,
                 a->h, a->f, (const float*)a->mod, a->block_size, D, nvec, a->out, a->skip_if);
    else
      launch_pdl(adaln_gated_residual_kernel<float>, dim3((unsigned)grid), dim3(kAdalnThreads), 0, stream, a->h,
                 a->f, (const float*)a->mod, a->block_size, D, nvec, a->out, a->skip_if);
  }
  return cudaGetLastError() == cudaSuccess ? TT_OK : TT_ERR_CUDA;
}

}  // namespace tt
