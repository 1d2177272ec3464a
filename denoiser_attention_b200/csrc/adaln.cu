// adaLN-single time conditioning on sm_100a: the paper §2.1 "Time conditioning" of
// "Nemotron-TwoTower: Diffusion Language Modeling with Pretrained AR Context" (adaLN-single as in
// PixArt-alpha: one global MLP from the diffusion time to shared shift/scale/gate, plus a learned
// per-layer embedding).
//
//   COND             tau -> mod[B][3][D]   three batched-GEMV launches (F->W, W->W, W->3D), each
//                                          reading its weight rows once for every sequence
//   NORM_MODULATE    RMSNorm prologue modulated by (shift, scale): one CTA per token row
//   GATED_RESIDUAL   h + gate * f: a vectorised elementwise pass
// All arithmetic is fp32 (the timestep sinusoid in fp64); bf16 tensors are widened on load and
// rounded to nearest on store.
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

// Batched GEMV for the three layers of the conditioning MLP:
//   y[b][o] = act(sum_i W[o][i] x[b][i] + bias[o]) (+ extra[o])
// Each warp holds R rows of W in registers (float4 per lane, KW of them per row) and applies them
// to every batch row; batch rows are staged in shared memory in chunks. kPhi: x is the timestep
// sinusoid phi(tau_b), computed in the kernel (IN = F); otherwise x is read from global memory.
constexpr int kGemvBatchChunk = 8;
constexpr int kGemvMaxIn = 1024;

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

template <int KW, int R, bool kPhi, bool kSilu>
__global__ void __launch_bounds__(kAdalnThreads) adaln_gemv_kernel(const float* __restrict__ Wt,
                                                                   const float* __restrict__ bias,
                                                                   const float* __restrict__ extra,
                                                                   const float* __restrict__ x, int B, int IN,
                                                                   int OUT, float* __restrict__ y) {
  __shared__ __align__(16) float s_x[kGemvBatchChunk * kGemvMaxIn];
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int o0 = (blockIdx.x * (kAdalnThreads / 32) + warp) * R;
  float4 w[R][KW];
  float bo[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int o = o0 + r;
    bo[r] = 0.f;
    if (o < OUT) bo[r] = bias[o] + (extra ? extra[o] : 0.f);
#pragma unroll
    for (int k = 0; k < KW; ++k) {
      const int i = (lane + 32 * k) * 4;
      w[r][k] = (o < OUT && i < IN) ? *reinterpret_cast<const float4*>(Wt + (size_t)o * IN + i)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  for (int b0 = 0; b0 < B; b0 += kGemvBatchChunk) {
    const int nb = min(kGemvBatchChunk, B - b0);
    __syncthreads();
    if (kPhi) {
      for (int bb = 0; bb < nb; ++bb) phi_row(x[b0 + bb], IN, s_x + bb * IN, threadIdx.x, blockDim.x);
    } else {
      for (int i = threadIdx.x; i < nb * IN; i += blockDim.x) s_x[i] = x[(size_t)b0 * IN + i];
    }
    __syncthreads();
    for (int bb = 0; bb < nb; ++bb) {
      float acc[R];
#pragma unroll
      for (int r = 0; r < R; ++r) acc[r] = 0.f;
#pragma unroll
      for (int k = 0; k < KW; ++k) {
        const int i = (lane + 32 * k) * 4;
        if (i < IN) {
          const float4 xv = *reinterpret_cast<const float4*>(s_x + bb * IN + i);
#pragma unroll
          for (int r = 0; r < R; ++r)
            acc[r] = fmaf(w[r][k].x, xv.x, fmaf(w[r][k].y, xv.y, fmaf(w[r][k].z, xv.z, fmaf(w[r][k].w, xv.w, acc[r]))));
        }
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float v = warp_sum(acc[r]) + bo[r];
        if (lane == 0 && o0 + r < OUT) y[(size_t)(b0 + bb) * OUT + o0 + r] = kSilu ? silu_f(v) : v;
      }
    }
  }
}

template <bool kPhi, bool kSilu>
static void launch_gemv(const float* Wt, const float* bias, const float* extra, const float* x, int B, int IN, int OUT,
                        float* y, cudaStream_t stream) {
  const int kw = (IN + 127) / 128;   // float4 per lane per row
  const int warps = kAdalnThreads / 32;
  // small layers: one row per warp (more CTAs); wide ones: four rows per warp
  const bool wide = OUT > 2048;
  if (kw <= 1) {
    if (wide)
      launch_pdl(adaln_gemv_kernel<1, 4, kPhi, kSilu>, dim3((OUT + warps * 4 - 1) / (warps * 4)), dim3(kAdalnThreads),
                 0, stream, Wt, bias, extra, x, B, IN, OUT, y);
    else
      launch_pdl(adaln_gemv_kernel<1, 1, kPhi, kSilu>, dim3((OUT + warps - 1) / warps), dim3(kAdalnThreads), 0,
                 stream, Wt, bias, extra, x, B, IN, OUT, y);
  } else if (kw <= 2) {
    if (wide)
      launch_pdl(adaln_gemv_kernel<2, 4, kPhi, kSilu>, dim3((OUT + warps * 4 - 1) / (warps * 4)), dim3(kAdalnThreads),
                 0, stream, Wt, bias, extra, x, B, IN, OUT, y);
    else
      launch_pdl(adaln_gemv_kernel<2, 1, kPhi, kSilu>, dim3((OUT + warps - 1) / warps), dim3(kAdalnThreads), 0,
                 stream, Wt, bias, extra, x, B, IN, OUT, y);
  } else if (kw <= 4) {
    launch_pdl(adaln_gemv_kernel<4, 1, kPhi, kSilu>, dim3((OUT + warps - 1) / warps), dim3(kAdalnThreads), 0, stream,
               Wt, bias, extra, x, B, IN, OUT, y);
  } else {
    launch_pdl(adaln_gemv_kernel<8, 1, kPhi, kSilu>, dim3((OUT + warps - 1) / warps), dim3(kAdalnThreads), 0, stream,
               Wt, bias, extra, x, B, IN, OUT, y);
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
                                                                            void* __restrict__ out) {
  constexpr int N = Io<T>::kN;
  pdl_trigger();
  pdl_wait();
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
                                                                             void* out) {
  constexpr int N = Io<T>::kN;
  pdl_trigger();
  pdl_wait();
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
  if (a->op == TT_ADALN_COND) return kHeaderBytes + 2 * sizeof(float) * (size_t)a->batch * a->mlp_width;
  return kHeaderBytes;
}

int adaln_launch(const tt_adaln_args_t* a, void* ws, cudaStream_t stream) {
  const int B = a->batch, D = a->hidden;
  if (a->op == TT_ADALN_COND) {
    float* a1 = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kHeaderBytes);
    float* a2 = a1 + (size_t)B * a->mlp_width;
    const int F = a->freq_dim, W = a->mlp_width;
    launch_gemv<true, true>(a->w1, a->b1, nullptr, a->tau, B, F, W, a1, stream);
    launch_gemv<false, true>(a->w2, a->b2, nullptr, a1, B, W, W, a2, stream);
    launch_gemv<false, false>(a->w3, a->b3, a->layer_emb, a2, B, W, 3 * D, a->mod, stream);
  } else if (a->op == TT_ADALN_NORM_MODULATE) {
    const int rows = B * a->block_size;
    if (a->dtype == TT_BF16)
      launch_pdl(adaln_norm_modulate_kernel<__nv_bfloat16>, dim3(rows), dim3(kAdalnThreads), 0, stream, a->h,
                 a->norm_w, (const float*)a->mod, a->block_size, D, a->eps, a->out);
    else
      launch_pdl(adaln_norm_modulate_kernel<float>, dim3(rows), dim3(kAdalnThreads), 0, stream, a->h, a->norm_w,
                 (const float*)a->mod, a->block_size, D, a->eps, a->out);
  } else {
    const int N = (a->dtype == TT_BF16) ? 8 : 4;
    const size_t nvec = (size_t)B * a->block_size * D / N;
    const int sms = device_sm_count();
    size_t grid = (nvec + kAdalnThreads - 1) / kAdalnThreads;
    grid = grid < (size_t)sms * 8 ? grid : (size_t)sms * 8;
    if (grid == 0) grid = 1;
    if (a->dtype == TT_BF16)
      launch_pdl(adaln_gated_residual_kernel<__nv_bfloat16>, dim3((unsigned)grid), dim3(kAdalnThreads), 0, stream,
                 a->h, a->f, (const float*)a->mod, a->block_size, D, nvec, a->out);
    else
      launch_pdl(adaln_gated_residual_kernel<float>, dim3((unsigned)grid), dim3(kAdalnThreads), 0, stream, a->h,
                 a->f, (const float*)a->mod, a->block_size, D, nvec, a->out);
  }
  return cudaGetLastError() == cudaSuccess ? TT_OK : TT_ERR_CUDA;
}

}  // namespace tt
