// adaLN-single time conditioning on sm_100a: the paper §2.1 "Time conditioning" of
// "Nemotron-TwoTower: Diffusion Language Modeling with Pretrained AR Context" (adaLN-single as in
// PixArt-alpha: one global MLP from the diffusion time to shared shift/scale/gate, plus a learned
// per-layer embedding).
//
//   COND             tau -> mod[B][3][D]   two launches: the small F->W->W part per sequence,
//                                          then the W->3D projection with W3 read once for all B
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

// Kernel A: per sequence b, phi(tau_b) -> a1 = SiLU(W1 phi + b1) -> a2 = SiLU(W2 a1 + b2).
__global__ void __launch_bounds__(kAdalnThreads) adaln_cond_hidden_kernel(const float* __restrict__ tau,
                                                                          const float* __restrict__ w1,
                                                                          const float* __restrict__ b1,
                                                                          const float* __restrict__ w2,
                                                                          const float* __restrict__ b2, int F,
                                                                          int W, float* __restrict__ a2_out) {
  __shared__ float s_phi[1024];
  __shared__ float s_a1[1024];
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int half = F / 2;
  const double t = 1000.0 * (double)tau[b];
  for (int k = tid; k < half; k += blockDim.x) {
    const double w = exp(-log(10000.0) * (double)k / (double)half);
    double sv, cv;
    sincos(t * w, &sv, &cv);
    s_phi[k] = (float)cv;
    s_phi[half + k] = (float)sv;
  }
  __syncthreads();
  const int nwarps = blockDim.x >> 5;
  for (int j = warp; j < W; j += nwarps) {
    const float* row = w1 + (size_t)j * F;
    float acc = 0.f;
    for (int i = lane; i < F; i += 32) acc = fmaf(row[i], s_phi[i], acc);
    acc = warp_sum(acc);
    if (lane == 0) s_a1[j] = silu_f(acc + b1[j]);
  }
  __syncthreads();
  for (int j = warp; j < W; j += nwarps) {
    const float* row = w2 + (size_t)j * W;
    float acc = 0.f;
    for (int i = lane; i < W; i += 32) acc = fmaf(row[i], s_a1[i], acc);
    acc = warp_sum(acc);
    if (lane == 0) a2_out[(size_t)b * W + j] = silu_f(acc + b2[j]);
  }
}

// Kernel B: mod[b][o] = W3[o] . a2[b] + b3[o] + emb[o] for o < 3D; one warp per output row o,
// reading the row once and reusing it for every sequence.
__global__ void __launch_bounds__(kAdalnThreads) adaln_cond_out_kernel(const float* __restrict__ a2,
                                                                       const float* __restrict__ w3,
                                                                       const float* __restrict__ b3,
                                                                       const float* __restrict__ emb, int B,
                                                                       int W, int out_rows,
                                                                       float* __restrict__ mod) {
  const int lane = threadIdx.x & 31;
  const int o = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (o >= out_rows) return;
  float wr[32];
  const float* row = w3 + (size_t)o * W;
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const int i = lane + 32 * k;
    wr[k] = (i < W) ? row[i] : 0.f;
  }
  const float bias = b3[o] + emb[o];
  for (int b = 0; b < B; ++b) {
    const float* x = a2 + (size_t)b * W;
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const int i = lane + 32 * k;
      if (i < W) acc = fmaf(wr[k], x[i], acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) mod[(size_t)b * out_rows + o] = acc + bias;
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
    adaln_cond_hidden_kernel<<<B, kAdalnThreads, 0, stream>>>(a->tau, a->w1, a->b1, a->w2, a->b2, a->freq_dim,
                                                              a->mlp_width, a2);
    const int rows = 3 * D;
    const int per_cta = kAdalnThreads / 32;
    adaln_cond_out_kernel<<<(rows + per_cta - 1) / per_cta, kAdalnThreads, 0, stream>>>(
        a2, a->w3, a->b3, a->layer_emb, B, a->mlp_width, rows, a->mod);
  } else if (a->op == TT_ADALN_NORM_MODULATE) {
    const int rows = B * a->block_size;
    if (a->dtype == TT_BF16)
      adaln_norm_modulate_kernel<__nv_bfloat16><<<rows, kAdalnThreads, 0, stream>>>(
          a->h, a->norm_w, a->mod, a->block_size, D, a->eps, a->out);
    else
      adaln_norm_modulate_kernel<float><<<rows, kAdalnThreads, 0, stream>>>(a->h, a->norm_w, a->mod,
                                                                            a->block_size, D, a->eps, a->out);
  } else {
    const int N = (a->dtype == TT_BF16) ? 8 : 4;
    const size_t nvec = (size_t)B * a->block_size * D / N;
    const int sms = device_sm_count();
    size_t grid = (nvec + kAdalnThreads - 1) / kAdalnThreads;
    grid = grid < (size_t)sms * 8 ? grid : (size_t)sms * 8;
    if (grid == 0) grid = 1;
    if (a->dtype == TT_BF16)
      adaln_gated_residual_kernel<__nv_bfloat16><<<(unsigned)grid, kAdalnThreads, 0, stream>>>(
          a->h, a->f, a->mod, a->block_size, D, nvec, a->out);
    else
      adaln_gated_residual_kernel<float><<<(unsigned)grid, kAdalnThreads, 0, stream>>>(
          a->h, a->f, a->mod, a->block_size, D, nvec, a->out);
  }
  return cudaGetLastError() == cudaSuccess ? TT_OK : TT_ERR_CUDA;
}

}  // namespace tt
