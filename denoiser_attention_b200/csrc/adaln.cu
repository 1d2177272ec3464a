// adaLN-single time conditioning on sm_100a: the paper §2.1 "Time conditioning" of
// "Nemotron-TwoTower: Diffusion Language Modeling with Pretrained AR Context" (adaLN-single as in
// PixArt-alpha: one global MLP from the diffusion time to shared shift/scale/gate, plus a learned
// per-layer embedding).
//
//   COND             tau -> mod[B][3][D]   three launches, one per layer (F->W with the sinusoid,
//                                          W->W, W->3D), each tiled over slices of 64 or 32
//                                          weight rows x chunks of 32, 16 or 8 sequences, operands
//                                          staged in shared memory with asynchronous copies
//   NORM_MODULATE    RMSNorm prologue modulated by (shift, scale): one warp per token row
//   GATED_RESIDUAL   h + gate * f: a vectorised elementwise pass
//   NORM_MODULATE_RESIDUAL  both from one read of h, in the RMSNorm kernel
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

// phi(tau) = [cos(1000 tau w_k), sin(1000 tau w_k)], w_k = 10000^(-k/(F/2)), for nb sequences
// (row bb of dst from tau[bb]). A thread computes its frequencies once and forms each sequence's
// angle (up to 1000 rad) and its reduction modulo 2 pi in double, so the single-precision sincos
// only sees |angle| <= pi.
__device__ __forceinline__ void phi_rows(const float* tau, int nb, int F, float* dst, int tid, int nthreads) {
  const int half = F / 2;
  const double two_pi = 6.283185307179586476925286766559;
  for (int k = tid; k < half; k += nthreads) {
    const double w = 1000.0 * exp(-9.2103403719761836 * (double)k / (double)half);   // ln(10000) = 9.2103...
    for (int bb = 0; bb < nb; ++bb) {
      double a = (double)tau[bb] * w;
      a -= two_pi * rint(a * (1.0 / two_pi));
      float sv, cv;
      sincosf((float)a, &sv, &cv);
      dst[bb * F + k] = cv;
      dst[bb * F + half + k] = sv;
    }
  }
}

constexpr int kMaxWidth = 1024;   // F and W bound (host-validated)

// 16-byte asynchronous copy global -> shared (L2 only); all of a stage's copies are in flight at
// once and completed with one wait.
__device__ __forceinline__ void cp_async16_g2s(void* smem, const void* gmem) {
  const uint32_t sa = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// One layer of the conditioning MLP for a slice of its outputs and a chunk of the sequences:
//   y[b][o] = act(W[o, :] . x_b + bias[o]) (+ extra[o]),  o in slice i, b in chunk j
// x_b is phi(tau_b) (kPhi: the timestep sinusoid, computed here) or row b of x. The CTA stages its
// 32 kRows rows of W (rows padded by 4 floats, so that the quarter-warp float4 reads of 8 rows hit
// distinct banks) and its chunk's input rows in shared memory with asynchronous copies; then a
// thread takes kRows output rows (lane, lane + 32, ...) for the kSeqPerWarp sequences of its warp,
// whose input rows are read as broadcasts: each float4 of W feeds kSeqPerWarp products and each
// float4 of x feeds kRows, which sets the ratio of arithmetic to shared-memory reads.
template <int kRows, int kSeqPerWarp>
struct RowsTile {
  static constexpr int kSlice = 32 * kRows;                           // output rows per CTA
  static constexpr int kChunk = kSeqPerWarp * (kAdalnThreads / 32);   // sequences per CTA
  static size_t smem_bytes(int IN) { return sizeof(float) * ((size_t)kSlice * (IN + 4) + (size_t)kChunk * IN); }
};

template <bool kPhi, bool kSilu, int kRows, int kSeqPerWarp>
__global__ void __launch_bounds__(kAdalnThreads) adaln_rows_kernel(const float* __restrict__ Wt,
                                                                   const float* __restrict__ bias,
                                                                   const float* __restrict__ extra,
                                                                   const float* __restrict__ x, int B, int IN,
                                                                   int OUT, float* __restrict__ y,
                                                                   const int32_t* skip_if) {
  using Tile = RowsTile<kRows, kSeqPerWarp>;
  extern __shared__ __align__(16) float s_dyn[];
  const int INP = IN + 4;
  float* s_w = s_dyn;                          // [kSlice][IN + 4]
  float* s_x = s_dyn + Tile::kSlice * INP;     // [kChunk][IN]
  pdl_trigger();
  pdl_wait();
  if (skip_requested(skip_if)) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int o0 = blockIdx.x * Tile::kSlice, b0 = blockIdx.y * Tile::kChunk;
  const int nrow = min(Tile::kSlice, OUT - o0), nb = min(Tile::kChunk, B - b0);
  const int iv = IN / 4;
  for (int i = threadIdx.x; i < nrow * iv; i += blockDim.x) {
    const int r = i / iv, c = i - r * iv;
    cp_async16_g2s(s_w + r * INP + 4 * c, Wt + (size_t)(o0 + r) * IN + 4 * c);
  }
  if (kPhi) {
    phi_rows(x + b0, nb, IN, s_x, threadIdx.x, blockDim.x);
  } else {
    for (int i = threadIdx.x; i < nb * iv; i += blockDim.x)
      cp_async16_g2s(s_x + 4 * i, x + (size_t)b0 * IN + 4 * i);
  }
  cp_async_wait_all();
  __syncthreads();
  const int bw = kSeqPerWarp * warp;   // this warp's first sequence of the chunk
  if (lane >= nrow || bw >= nb) return;
  float acc[kRows][kSeqPerWarp];
#pragma unroll
  for (int r = 0; r < kRows; ++r)
#pragma unroll
    for (int q = 0; q < kSeqPerWarp; ++q) acc[r][q] = 0.f;
  // rows past the slice's end read a valid staged row (row 0); their results are not stored
  const float* wrow[kRows];
#pragma unroll
  for (int r = 0; r < kRows; ++r) wrow[r] = s_w + (lane + 32 * r < nrow ? lane + 32 * r : 0) * INP;
  const float* xrow[kSeqPerWarp];
#pragma unroll
  for (int q = 0; q < kSeqPerWarp; ++q) xrow[q] = s_x + (bw + q < nb ? bw + q : bw) * IN;
  for (int k = 0; k < IN; k += 4) {
    float4 wv[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) wv[r] = *reinterpret_cast<const float4*>(wrow[r] + k);
#pragma unroll
    for (int q = 0; q < kSeqPerWarp; ++q) {
      const float4 u = *reinterpret_cast<const float4*>(xrow[q] + k);
#pragma unroll
      for (int r = 0; r < kRows; ++r)
        acc[r][q] = fmaf(wv[r].x, u.x, fmaf(wv[r].y, u.y, fmaf(wv[r].z, u.z, fmaf(wv[r].w, u.w, acc[r][q]))));
    }
  }
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    if (lane + 32 * r >= nrow) break;
    const int o = o0 + lane + 32 * r;
    const float add = bias[o] + (extra ? extra[o] : 0.f);
#pragma unroll
    for (int q = 0; q < kSeqPerWarp; ++q) {
      if (bw + q < nb) {
        float v = acc[r][q] + add;
        if (kSilu) v = silu_f(v);
        y[(size_t)(b0 + bw + q) * OUT + o] = v;
      }
    }
  }
}

// Tile choice: 64 rows x 32 sequences (2 rows and 4 sequences per thread) when the staged rows fit
// in kWideTileSmem (inputs up to 256 wide) and the grid still has at least one CTA per SM (the
// 6144-row output layer); else 32 rows x 16 or 8 sequences, the wider while it fills the SMs, so
// that narrow layers (few row slices) spread over more CTAs.
constexpr size_t kWideTileSmem = 100 * 1024;
constexpr int kFillCtas = 148;

template <bool kPhi, bool kSilu, int kRows, int kSeqPerWarp>
static cudaError_t launch_rows_tile(const float* Wt, const float* bias, const float* extra, const float* x, int B,
                                    int IN, int OUT, float* y, const int32_t* skip_if, cudaStream_t stream) {
  using Tile = RowsTile<kRows, kSeqPerWarp>;
  const dim3 grid((OUT + Tile::kSlice - 1) / Tile::kSlice, (B + Tile::kChunk - 1) / Tile::kChunk);
  return launch_pdl(adaln_rows_kernel<kPhi, kSilu, kRows, kSeqPerWarp>, grid, dim3(kAdalnThreads),
                    Tile::smem_bytes(IN), stream, Wt, bias, extra, x, B, IN, OUT, y, skip_if);
}

template <int kRows, int kSeqPerWarp>
static long long tile_ctas(int B, int OUT) {
  using Tile = RowsTile<kRows, kSeqPerWarp>;
  return (long long)((OUT + Tile::kSlice - 1) / Tile::kSlice) * ((B + Tile::kChunk - 1) / Tile::kChunk);
}

template <bool kPhi, bool kSilu>
static cudaError_t launch_rows(const float* Wt, const float* bias, const float* extra, const float* x, int B, int IN,
                               int OUT, float* y, const int32_t* skip_if, cudaStream_t stream) {
  if (RowsTile<2, 4>::smem_bytes(IN) <= kWideTileSmem && tile_ctas<2, 4>(B, OUT) >= kFillCtas)
    return launch_rows_tile<kPhi, kSilu, 2, 4>(Wt, bias, extra, x, B, IN, OUT, y, skip_if, stream);
  if (tile_ctas<1, 2>(B, OUT) >= kFillCtas)
    return launch_rows_tile<kPhi, kSilu, 1, 2>(Wt, bias, extra, x, B, IN, OUT, y, skip_if, stream);
  return launch_rows_tile<kPhi, kSilu, 1, 1>(Wt, bias, extra, x, B, IN, OUT, y, skip_if, stream);
}

template <bool kPhi, bool kSilu, int kRows, int kSeqPerWarp>
static bool set_rows_smem(int bytes) {
  return cudaFuncSetAttribute(adaln_rows_kernel<kPhi, kSilu, kRows, kSeqPerWarp>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
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

// 8 consecutive floats (a 16-byte aligned address) into x[0..7], or 4 into x[0..3] (kN == 4)
template <int kN>
__device__ __forceinline__ void load_f32(const float* p, float* x) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  if constexpr (kN == 8) {
    const float4 c = *reinterpret_cast<const float4*>(p + 4);
    x[4] = c.x; x[5] = c.y; x[6] = c.z; x[7] = c.w;
  }
}

// One warp per token row (b, s): y = h / sqrt(mean(h^2) + eps) * w * (1 + scale_b) + shift_b. A
// lane keeps up to kNormVec of its row's vectors in registers from the sum of squares to the
// output (one read of h for rows up to 32 kNormVec vectors: D <= 2048 in bf16), the sum is a
// warp-shuffle reduction, and w, scale and shift are read as float4. With kResid the same pass
// also writes out2 = h + gate_b * f, from the h already loaded: the vectors held in registers get
// it while the sum of squares is formed, those of wider rows when they are read again for y (so
// out2 may alias h).
constexpr int kNormVec = 8;
constexpr int kNormRowsPerCta = 4;

template <typename T, bool kResid>
__global__ void __launch_bounds__(32 * kNormRowsPerCta) adaln_norm_modulate_kernel(const void* __restrict__ h,
                                                                                   const float* __restrict__ norm_w,
                                                                                   const float* __restrict__ mod,
                                                                                   const void* __restrict__ f,
                                                                                   int rows, int S, int D, float eps,
                                                                                   void* __restrict__ out,
                                                                                   void* out2,
                                                                                   const int32_t* skip_if) {
  constexpr int N = Io<T>::kN;
  pdl_trigger();
  pdl_wait();
  if (skip_requested(skip_if)) return;
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kNormRowsPerCta + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int b = row / S;
  const int nv = D / N;
  const size_t vbase = (size_t)row * nv;
  const float* shift = mod + (size_t)b * 3 * D;
  const float* scale = shift + D;
  const float* gate = shift + 2 * D;
  // out2 = h + gate * f for vector v whose h is x
  auto residual = [&](int v, const float* x) {
    float fv[N], g[N], o[N];
    Io<T>::load(f, vbase + v, fv);
    load_f32<N>(gate + v * N, g);
#pragma unroll
    for (int k = 0; k < N; ++k) o[k] = fmaf(g[k], fv[k], x[k]);
    Io<T>::store(out2, vbase + v, o);
  };
  float xr[kNormVec][N];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kNormVec; ++i) {
    const int v = lane + 32 * i;
    if (v < nv) {
      Io<T>::load(h, vbase + v, xr[i]);
#pragma unroll
      for (int k = 0; k < N; ++k) ss = fmaf(xr[i][k], xr[i][k], ss);
      if constexpr (kResid) residual(v, xr[i]);
    }
  }
  for (int v = lane + 32 * kNormVec; v < nv; v += 32) {   // rows wider than the register cache
    float x[N];
    Io<T>::load(h, vbase + v, x);
#pragma unroll
    for (int k = 0; k < N; ++k) ss = fmaf(x[k], x[k], ss);
  }
  const float r = 1.0f / sqrtf(warp_sum(ss) / (float)D + eps);
  auto emit = [&](int v, float* x) {
    const int j0 = v * N;
    float w[N], sc[N], sh[N];
    load_f32<N>(norm_w + j0, w);
    load_f32<N>(scale + j0, sc);
    load_f32<N>(shift + j0, sh);
#pragma unroll
    for (int k = 0; k < N; ++k) x[k] = fmaf(x[k] * r * w[k], 1.0f + sc[k], sh[k]);
    Io<T>::store(out, vbase + v, x);
  };
#pragma unroll
  for (int i = 0; i < kNormVec; ++i) {
    const int v = lane + 32 * i;
    if (v < nv) emit(v, xr[i]);
  }
  for (int v = lane + 32 * kNormVec; v < nv; v += 32) {
    float x[N];
    Io<T>::load(h, vbase + v, x);
    if constexpr (kResid) residual(v, x);
    emit(v, x);
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
    float x[N], y[N], g[N];
    Io<T>::load(h, v, x);
    Io<T>::load(f, v, y);
    load_f32<N>(mod + (size_t)b * 3 * D + 2 * D + j0, g);
#pragma unroll
    for (int k = 0; k < N; ++k) x[k] = fmaf(g[k], y[k], x[k]);
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
    const int F = a->freq_dim, W = a->mlp_width, OUT = 3 * D;
    // the shared-memory opt-in for inputs up to kMaxWidth wide, once per device (so that no
    // attribute call happens while a caller captures the stream into a CUDA graph)
    static unsigned long long attr_done = 0;   // bit per device ordinal (< 64)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return TT_ERR_CUDA;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(__atomic_load_n(&attr_done, __ATOMIC_ACQUIRE) & bit)) {
      const int sw = (int)kWideTileSmem, s2 = (int)RowsTile<1, 2>::smem_bytes(kMaxWidth),
                s1 = (int)RowsTile<1, 1>::smem_bytes(kMaxWidth);
      if (!set_rows_smem<true, true, 2, 4>(sw) || !set_rows_smem<false, true, 2, 4>(sw) ||
          !set_rows_smem<false, false, 2, 4>(sw) || !set_rows_smem<true, true, 1, 2>(s2) ||
          !set_rows_smem<false, true, 1, 2>(s2) || !set_rows_smem<false, false, 1, 2>(s2) ||
          !set_rows_smem<true, true, 1, 1>(s1) || !set_rows_smem<false, true, 1, 1>(s1) ||
          !set_rows_smem<false, false, 1, 1>(s1))
        return TT_ERR_CUDA;
      __atomic_fetch_or(&attr_done, bit, __ATOMIC_ACQ_REL);
    }
    if (launch_rows<true, true>(a->w1, a->b1, nullptr, a->tau, B, F, W, a1, a->skip_if, stream) != cudaSuccess ||
        launch_rows<false, true>(a->w2, a->b2, nullptr, a1, B, W, W, a2, a->skip_if, stream) != cudaSuccess ||
        launch_rows<false, false>(a->w3, a->b3, a->layer_emb, a2, B, W, OUT, a->mod, a->skip_if, stream) !=
            cudaSuccess)
      return TT_ERR_CUDA;
  } else if (a->op == TT_ADALN_NORM_MODULATE || a->op == TT_ADALN_NORM_MODULATE_RESIDUAL) {
    const int rows = B * a->block_size;
    const dim3 grid((rows + kNormRowsPerCta - 1) / kNormRowsPerCta), block(32 * kNormRowsPerCta);
    const bool resid = (a->op == TT_ADALN_NORM_MODULATE_RESIDUAL);
    const float* mod = a->mod;
    cudaError_t e;
    if (a->dtype == TT_BF16)
      e = resid ? launch_pdl(adaln_norm_modulate_kernel<__nv_bfloat16, true>, grid, block, 0, stream, a->h,
                             a->norm_w, mod, a->f, rows, a->block_size, D, a->eps, a->out, a->out2, a->skip_if)
                : launch_pdl(adaln_norm_modulate_kernel<__nv_bfloat16, false>, grid, block, 0, stream, a->h,
                             a->norm_w, mod, a->f, rows, a->block_size, D, a->eps, a->out, a->out2, a->skip_if);
    else
      e = resid ? launch_pdl(adaln_norm_modulate_kernel<float, true>, grid, block, 0, stream, a->h, a->norm_w, mod,
                             a->f, rows, a->block_size, D, a->eps, a->out, a->out2, a->skip_if)
                : launch_pdl(adaln_norm_modulate_kernel<float, false>, grid, block, 0, stream, a->h, a->norm_w,
                             mod, a->f, rows, a->block_size, D, a->eps, a->out, a->out2, a->skip_if);
    if (e != cudaSuccess) return TT_ERR_CUDA;
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
