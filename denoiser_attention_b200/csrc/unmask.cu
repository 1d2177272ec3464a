// ConfidenceSample on sm_100a: the paper §2.2 "Sampling" and Algorithm 2 line 5 of
// "Nemotron-TwoTower: Diffusion Language Modeling with Pretrained AR Context".
//
// One pass over the vocabulary logits computes, per block position, the softmax maximum
// probability (confidence) and the argmax token; the CTA that finishes the last position of a
// sequence then applies the commit rule to that sequence. Logits are read once, with 128-bit
// streaming loads, 8 in flight per thread.
//
// Work split: the logits of all positions are one flat array of 16-byte vectors, cut into equal
// contiguous ranges, one per CTA (4 CTAs per SM), so every SM streams the same number of bytes
// whatever the vocabulary size. A range covers the tail of one position and the head of the next
// at most a few times; a position cut between CTAs is finished by the last of them to arrive (an
// atomic ticket; no spinning), which merges the per-CTA partial states. Per thread the running
// state is (m, s, idx): the largest raw logit seen, s = sum exp(c (x - m)) with
// c = inv_temperature * log2(e) evaluated as exp2, and the lowest index attaining m. States merge
// associatively; ties keep the lower token index at every level.
#include <cmath>
#include <cstdio>
#include <algorithm>
#include <mutex>

#include "tt_common.cuh"
#include "tt_internal.h"

namespace tt {

struct UnmaskPartial {
  float m;
  float s;
  int32_t idx;
  int32_t pad;
};

struct RedState {
  float m;
  float s;
  int32_t idx;
};

__device__ __forceinline__ RedState red_combine(RedState a, RedState b, float c) {
  RedState r;
  const bool take_b = (b.m > a.m) || (b.m == a.m && b.idx < a.idx);
  r.idx = take_b ? b.idx : a.idx;
  r.m = fmaxf(a.m, b.m);
  const float sa = (a.m == -INFINITY) ? 0.f : a.s * ex2(c * (a.m - r.m));
  const float sb = (b.m == -INFINITY) ? 0.f : b.s * ex2(c * (b.m - r.m));
  r.s = sa + sb;
  return r;
}

template <typename T>
struct VecTraits;
template <>
struct VecTraits<float> {
  static constexpr int kN = 4;
  __device__ static void to_float(const uint4& v, float* x) {
    x[0] = __uint_as_float(v.x);
    x[1] = __uint_as_float(v.y);
    x[2] = __uint_as_float(v.z);
    x[3] = __uint_as_float(v.w);
  }
};
template <>
struct VecTraits<__nv_bfloat16> {
  static constexpr int kN = 8;
  __device__ static void to_float(const uint4& v, float* x) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};

struct UnmaskParams {
  const void* logits;
  int32_t vocab;
  int32_t vec_per_row;   // vocab / vector width
  long long total_vec;   // rows * vec_per_row
  long long p_eff;       // working CTAs = min(gridDim.x, total_vec)
  int32_t rows;          // B*S
  int32_t block_size;    // S
  float c;               // inv_temperature * log2(e)
  float gamma;
  int32_t mask_token_id;
  int32_t exclude_mask_token;
  int32_t remaining_steps;
  int32_t sampler;           // tt_sampler_t
  int32_t keep_masked;
  int32_t* tokens;
  uint8_t* is_masked;
  float* conf_out;
  int32_t* argmax_out;
  int32_t* n_committed;
  int32_t* n_masked;
  uint8_t* ws;
  size_t off_row_cnt, off_seq_cnt, off_partials, off_conf, off_argmax;
};

constexpr int kUnmaskThreads = 256;
constexpr int kUnmaskUnroll = 8;
constexpr int kUnmaskCtasPerSm = 4;

// CTA owning vector v when E vectors are cut into P <= E ranges [c*E/P, (c+1)*E/P).
__device__ __forceinline__ long long owner_of(long long v, long long E, long long P) {
  return ((v + 1) * P - 1) / E;
}

// Commit rule for one sequence, run by the whole CTA.
__device__ void commit_sequence(const UnmaskParams& p, int b, const float* conf_ws, const int32_t* arg_ws) {
  __shared__ float s_conf[1024];
  __shared__ uint8_t s_masked[1024];
  __shared__ int s_counts[2];
  const int S = p.block_size;
  const int tid = threadIdx.x;
  if (tid < 2) s_counts[tid] = 0;
  __syncthreads();
  int my_masked = 0, my_ge = 0;
  for (int l = tid; l < S; l += blockDim.x) {
    const float cf = __ldcg(conf_ws + (size_t)b * S + l);
    const uint8_t mk = p.is_masked[(size_t)b * S + l] ? 1 : 0;
    s_conf[l] = cf;
    s_masked[l] = mk;
    my_masked += mk;
    my_ge += (mk && cf >= p.gamma) ? 1 : 0;
  }
  atomicAdd(&s_counts[0], my_masked);
  atomicAdd(&s_counts[1], my_ge);
  __syncthreads();
  const int n_masked = s_counts[0];
  const int n_ge = s_counts[1];
  int K;
  if (p.sampler == TT_SAMPLER_PREDICT_NOISE) {
    // predict-and-noise: all but keep_masked of the masked positions are committed
    K = max(0, n_masked - p.keep_masked);
  } else {
    int need = 0;
    if (n_masked > 0) need = (p.remaining_steps > 0) ? (n_masked + p.remaining_steps - 1) / p.remaining_steps : 1;
    K = max(need, n_ge);
  }
  // a masked position commits iff its rank among masked positions (confidence descending,
  // position ascending) is below K; every position >= gamma ranks below n_ge <= K.
  for (int l = tid; l < S; l += blockDim.x) {
    if (!s_masked[l]) continue;
    const float cl = s_conf[l];
    int rank = 0;
    for (int j = 0; j < S; ++j) {
      if (!s_masked[j]) continue;
      const float cj = s_conf[j];
      rank += (cj > cl || (cj == cl && j < l)) ? 1 : 0;
    }
    if (rank < K) {
      p.tokens[(size_t)b * S + l] = __ldcg(arg_ws + (size_t)b * S + l);
      p.is_masked[(size_t)b * S + l] = 0;
    }
  }
  if (tid == 0) {
    const int committed = min(K, n_masked);
    p.n_committed[b] = committed;
    p.n_masked[b] = n_masked - committed;
  }
}

template <typename T>
__global__ void __launch_bounds__(kUnmaskThreads) unmask_kernel(const UnmaskParams p) {
  using VT = VecTraits<T>;
  constexpr int N = VT::kN;
  pdl_trigger();
  pdl_wait();
  const long long cta = blockIdx.x;
  if (cta >= p.p_eff) return;
  const int tid = threadIdx.x;
  const float c = p.c;
  const long long E = p.total_vec, Pe = p.p_eff;
  const long long vbeg = cta * E / Pe, vend = (cta + 1) * E / Pe;
  const uint4* base = reinterpret_cast<const uint4*>(p.logits);

  float* conf_ws = reinterpret_cast<float*>(p.ws + p.off_conf);
  int32_t* arg_ws = reinterpret_cast<int32_t*>(p.ws + p.off_argmax);
  int* row_cnt = reinterpret_cast<int*>(p.ws + p.off_row_cnt);
  int* seq_cnt = reinterpret_cast<int*>(p.ws + p.off_seq_cnt);
  UnmaskPartial* parts = reinterpret_cast<UnmaskPartial*>(p.ws + p.off_partials);
  __shared__ RedState s_red[kUnmaskThreads / 32];
  __shared__ int s_flag;
  const int warp = tid >> 5, lane = tid & 31;

  for (long long seg = vbeg; seg < vend;) {
    const int row = (int)(seg / p.vec_per_row);
    const long long row_beg = (long long)row * p.vec_per_row;
    const long long seg_end = min(vend, row_beg + p.vec_per_row);
    const int vb = (int)(seg - row_beg), ve = (int)(seg_end - row_beg);   // vectors of this row
    const uint4* vp = base + row_beg;

    float m = -INFINITY, s = 0.f;
    int32_t idx = 0x7fffffff;
    auto consume = [&](const uint4& raw, int vi_global) {
      const int vbase = vi_global * N;
      float x[N];
      VT::to_float(raw, x);
      if (p.exclude_mask_token) {
        const int r = p.mask_token_id - vbase;
#pragma unroll
        for (int k = 0; k < N; ++k)   // static indices keep x[] in registers
          if (k == r) x[k] = -INFINITY;
      }
      float vm = x[0];
      int vi = 0;
#pragma unroll
      for (int k = 1; k < N; ++k) {
        if (x[k] > vm) { vm = x[k]; vi = k; }
      }
      if (vm > m) {
        s = (m == -INFINITY) ? 0.f : s * ex2(c * (m - vm));
        m = vm;
        idx = vbase + vi;
      }
      const float nmc = -c * m;
#pragma unroll
      for (int k = 0; k < N; ++k) s += ex2(fmaf(x[k], c, nmc));
    };
    int v = vb + tid;
    for (; v + (kUnmaskUnroll - 1) * kUnmaskThreads < ve; v += kUnmaskUnroll * kUnmaskThreads) {
      uint4 raw[kUnmaskUnroll];
#pragma unroll
      for (int u = 0; u < kUnmaskUnroll; ++u) raw[u] = __ldcs(vp + v + u * kUnmaskThreads);
#pragma unroll
      for (int u = 0; u < kUnmaskUnroll; ++u) consume(raw[u], v + u * kUnmaskThreads);
    }
    for (; v < ve; v += kUnmaskThreads) consume(__ldcs(vp + v), v);

    // ---- CTA reduction (warp shuffles, then across warps), lowest index on ties
    RedState st{m, s, idx};
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      RedState o;
      o.m = __shfl_xor_sync(0xffffffffu, st.m, off);
      o.s = __shfl_xor_sync(0xffffffffu, st.s, off);
      o.idx = __shfl_xor_sync(0xffffffffu, st.idx, off);
      st = red_combine(st, o, c);
    }
    __syncthreads();   // s_red / s_flag reuse across segments
    if (lane == 0) s_red[warp] = st;
    __syncthreads();
    if (tid == 0) {
      RedState r = s_red[0];
      for (int w = 1; w < kUnmaskThreads / 32; ++w) r = red_combine(r, s_red[w], c);
      const long long c_lo = owner_of(row_beg, E, Pe), c_hi = owner_of(row_beg + p.vec_per_row - 1, E, Pe);
      bool row_done = true;
      if (c_hi > c_lo) {
        const size_t slot = (size_t)row + (size_t)cta;   // unique per (row, CTA) pair
        parts[slot] = UnmaskPartial{r.m, r.s, r.idx, 0};
        __threadfence();
        const int old = atomicAdd(row_cnt + row, 1);
        row_done = (old == (int)(c_hi - c_lo));
        if (row_done) {
          row_cnt[row] = 0;
          __threadfence();
          const float4* pp = reinterpret_cast<const float4*>(parts);
          float4 q = __ldcg(pp + (size_t)row + (size_t)c_lo);
          r = RedState{q.x, q.y, __float_as_int(q.z)};
          for (long long k = c_lo + 1; k <= c_hi; ++k) {
            q = __ldcg(pp + (size_t)row + (size_t)k);
            r = red_combine(r, RedState{q.x, q.y, __float_as_int(q.z)}, c);
          }
        }
      }
      int last_of_seq = 0;
      if (row_done) {
        const float conf = 1.0f / r.s;
        conf_ws[row] = conf;
        arg_ws[row] = r.idx;
        if (p.conf_out) p.conf_out[row] = conf;
        if (p.argmax_out) p.argmax_out[row] = r.idx;
        __threadfence();
        const int b = row / p.block_size;
        const int old = atomicAdd(seq_cnt + b, 1);
        if (old == p.block_size - 1) {
          seq_cnt[b] = 0;
          __threadfence();
          last_of_seq = 1;
        }
      }
      s_flag = last_of_seq;
    }
    __syncthreads();
    if (s_flag) commit_sequence(p, row / p.block_size, conf_ws, arg_ws);
    seg = seg_end;
  }
}

static UnmaskLayout layout_for(int rows, int batch, int grid) {
  UnmaskLayout L{};
  size_t off = kHeaderBytes;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = (off + bytes + 255) & ~size_t(255);
    return o;
  };
  L.row_cnt = take(sizeof(int) * (size_t)rows);
  L.seq_cnt = take(sizeof(int) * (size_t)batch);
  L.partials = take(sizeof(UnmaskPartial) * ((size_t)rows + (size_t)grid));
  L.conf = take(sizeof(float) * (size_t)rows);
  L.argmax = take(sizeof(int32_t) * (size_t)rows);
  L.total = off;
  return L;
}

UnmaskPlan unmask_plan(const tt_unmask_args_t* a, int num_sms) {
  UnmaskPlan pl{};
  const int rows = a->batch * a->block_size;
  const int W = (a->dtype == TT_BF16) ? 8 : 4;
  const long long E = (long long)rows * (a->vocab / W);
  const long long P = (long long)std::max(num_sms, 1) * kUnmaskCtasPerSm;
  pl.grid = (int)std::min(P, E);
  pl.layout = layout_for(rows, a->batch, pl.grid);
  return pl;
}

int unmask_launch(const tt_unmask_args_t* a, const UnmaskPlan& pl, void* ws, cudaStream_t stream) {
  UnmaskParams p{};
  const int W = (a->dtype == TT_BF16) ? 8 : 4;
  p.logits = a->logits;
  p.vocab = a->vocab;
  p.vec_per_row = a->vocab / W;
  p.rows = a->batch * a->block_size;
  p.total_vec = (long long)p.rows * p.vec_per_row;
  p.p_eff = pl.grid;
  p.block_size = a->block_size;
  p.c = a->inv_temperature * 1.4426950408889634f;
  p.gamma = a->gamma;
  p.mask_token_id = a->mask_token_id;
  p.exclude_mask_token = a->exclude_mask_token;
  p.remaining_steps = a->remaining_steps;
  p.sampler = a->sampler;
  p.keep_masked = a->keep_masked;
  p.tokens = a->tokens;
  p.is_masked = a->is_masked;
  p.conf_out = a->conf;
  p.argmax_out = a->argmax;
  p.n_committed = a->n_committed;
  p.n_masked = a->n_masked;
  p.ws = static_cast<uint8_t*>(ws);
  p.off_row_cnt = pl.layout.row_cnt;
  p.off_seq_cnt = pl.layout.seq_cnt;
  p.off_partials = pl.layout.partials;
  p.off_conf = pl.layout.conf;
  p.off_argmax = pl.layout.argmax;
  if (a->dtype == TT_BF16)
    launch_pdl(unmask_kernel<__nv_bfloat16>, dim3(pl.grid), dim3(kUnmaskThreads), 0, stream, p);
  else
    launch_pdl(unmask_kernel<float>, dim3(pl.grid), dim3(kUnmaskThreads), 0, stream, p);
  return cudaGetLastError() == cudaSuccess ? TT_OK : TT_ERR_CUDA;
}

// ---------------------------------------------------------------- no-allocation variant
// The same kernel and launch as above, but its scratch is a fixed-size array in this module's
// static device memory instead of a caller workspace. It serves callers that cannot allocate
// device memory at the point of the call: a host runtime that has no CUDA allocator of its own
// (it owns only the logits/token buffers handed to it), or a thread that must not enter an
// allocator (e.g. one running under an allocator lock, or a real-time decode loop that forbids
// allocation after start-up).
//
// The layout is the one layout_for() gives for the largest supported sizes, fixed once, so its
// offsets never move between calls of different sizes; the kernel returns the merge tickets it
// uses to zero, so after the one clearing at setup every later call finds them at zero.
constexpr int kStaticMaxRows = 4096;   // batch * block_size
constexpr int kStaticMaxGrid = 1024;   // CTAs (partial slots beyond the rows)
constexpr size_t kStaticScratchBytes = 168 * 1024;

static __device__ __align__(256) uint8_t g_unmask_scratch[kStaticScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
uint8_t* g_static_ptr[kMaxDevices] = {};
}  // namespace

int unmask_launch_static(const tt_unmask_args_t* a, cudaStream_t stream) {
  const int rows = a->batch * a->block_size;
  if (rows > kStaticMaxRows) return TT_ERR_WORKSPACE_TOO_SMALL;
  const UnmaskLayout L = layout_for(kStaticMaxRows, kStaticMaxRows, kStaticMaxGrid);
  if (L.total > kStaticScratchBytes) return TT_ERR_WORKSPACE_TOO_SMALL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TT_ERR_CUDA;
  uint8_t* ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_static_mu);
    ws = g_static_ptr[dev];
    if (!ws) {
      // Setup, once per device, with that device current: resolve the array's address and clear
      // the header and the ticket counters (everything before the partial slots), stream-ordered
      // before the first launch.
      void* sym = nullptr;
      if (cudaGetSymbolAddress(&sym, g_unmask_scratch) != cudaSuccess || !sym) return TT_ERR_CUDA;
      if (cudaMemsetAsync(sym, 0, L.partials, stream) != cudaSuccess) return TT_ERR_CUDA;
      ws = static_cast<uint8_t*>(sym);
      g_static_ptr[dev] = ws;
    }
  }
  UnmaskPlan pl = unmask_plan(a, device_sm_count());
  pl.grid = std::min(pl.grid, kStaticMaxGrid);
  pl.layout = L;
  return unmask_launch(a, pl, ws, stream);
}

// ---------------------------------------------------------------- Algorithm 2 line 3
// tau_b = |{l : position l of sequence b is masked}| / S, one warp per sequence, so a multi-step
// refinement loop can feed the next step's time input from the mask on the device.
constexpr int kTauThreads = 128;

__global__ void __launch_bounds__(kTauThreads) block_tau_kernel(const uint8_t* __restrict__ is_masked, int B, int S,
                                                                float* __restrict__ tau) {
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x * (kTauThreads / 32) + warp;
  if (b >= B) return;
  int n = 0;
  for (int l = lane; l < S; l += 32) n += is_masked[(size_t)b * S + l] ? 1 : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
  if (lane == 0) tau[b] = (float)n / (float)S;
}

int block_tau_launch(const uint8_t* is_masked, int B, int S, float* tau, cudaStream_t stream) {
  const int per = kTauThreads / 32;
  return launch_pdl(block_tau_kernel, dim3((B + per - 1) / per), dim3(kTauThreads), 0, stream, is_masked, B, S, tau) ==
                 cudaSuccess
             ? TT_OK
             : TT_ERR_CUDA;
}

}  // namespace tt
