// ConfidenceSample on sm_100a: the paper §2.2 "Sampling" and Algorithm 2 (its ConfidenceSample step) of
// "Nemotron-TwoTower: Diffusion Language Modeling with Pretrained AR Context".
//
// One pass over the vocabulary logits computes, per block position, the softmax maximum
// probability (confidence) and the argmax token; the CTA that finishes the last position of a
// sequence then applies the commit rule to that sequence. Logits are read once: each thread
// streams its 16-byte vectors through its own ring of 8 shared-memory slots with asynchronous
// copies (cp.async, L2 only), so 8 loads stay in flight per thread without holding registers and
// without block barriers.
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
#include <cuda.h>
#include <cudaTypedefs.h>

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
  int32_t batch;               // B
  size_t off_done;             // 64-bit word: (sequences committed << 32) + masked positions left
  const int32_t* skip_if;      // early exit of a loop: non-zero => do nothing
  int32_t* all_done;           // set to 1 when no sequence has a masked position left
};

constexpr int kUnmaskThreads = 256;
constexpr int kUnmaskRing = 8;    // 16-byte vectors in flight per thread (shared-memory ring)
constexpr int kUnmaskCtasPerSm = 4;

// CTA owning vector v when E vectors are cut into P <= E ranges [c*E/P, (c+1)*E/P).
__device__ __forceinline__ long long owner_of(long long v, long long E, long long P) {
  return ((v + 1) * P - 1) / E;
}

// Commit rule for one sequence, run by the whole CTA.
// blocks up to this many positions rank by counting; longer ones sort
constexpr int kRankLoopMax = 64;

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
  if (S <= kRankLoopMax) {
    // short blocks: each thread counts its positions' ranks directly (S comparisons each)
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
  } else {
    // long blocks: a bitonic sort of 64-bit keys (confidence descending in the high word,
    // position ascending in the low word; unmasked positions and the padding to a power of two
    // sort last), then the first K sorted positions commit
    __shared__ unsigned long long s_key[1024];
    int P = 1;
    while (P < S) P <<= 1;
    for (int l = tid; l < P; l += blockDim.x) {
      unsigned long long key = ~0ull;
      if (l < S && s_masked[l]) {
        const uint32_t u = __float_as_uint(s_conf[l]);
        const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);   // ascending in the float's order
        key = ((unsigned long long)(~ord) << 32) | (uint32_t)l;
      }
      s_key[l] = key;
    }
    __syncthreads();
    for (int k = 2; k <= P; k <<= 1) {
      for (int jd = k >> 1; jd > 0; jd >>= 1) {
        for (int i = tid; i < P; i += blockDim.x) {
          const int ix = i ^ jd;
          if (ix > i) {
            const unsigned long long x = s_key[i], y = s_key[ix];
            if ((x > y) == ((i & k) == 0)) {
              s_key[i] = y;
              s_key[ix] = x;
            }
          }
        }
        __syncthreads();
      }
    }
    for (int r = tid; r < min(K, n_masked); r += blockDim.x) {
      const int l = (int)(uint32_t)(s_key[r] & 0xffffffffull);
      p.tokens[(size_t)b * S + l] = __ldcg(arg_ws + (size_t)b * S + l);
      p.is_masked[(size_t)b * S + l] = 0;
    }
  }
  if (tid == 0) {
    const int committed = min(K, n_masked);
    p.n_committed[b] = committed;
    p.n_masked[b] = n_masked - committed;
    if (p.all_done) {
      // one 64-bit ticket counts the committed sequences (high half) and sums their masked
      // positions left (low half); the last sequence reads the total, returns the word to zero
      // and raises the loop's done word when nothing is left masked
      unsigned long long* word = reinterpret_cast<unsigned long long*>(p.ws + p.off_done);
      const unsigned long long left = (unsigned long long)(unsigned)(n_masked - committed);
      const unsigned long long old = atomicAdd(word, (1ull << 32) | left);
      if ((old >> 32) == (unsigned long long)(p.batch - 1)) {
        const unsigned long long total = (old & 0xffffffffull) + left;
        *word = 0ull;
        if (total == 0) *p.all_done = 1;
      }
    }
  }
}

// 16-byte asynchronous copy global -> shared (L2 only), one commit group per call site
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t sa = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// atomicAdd with acquire-release semantics at GPU scope: the writes before it are visible to a
// thread that later acquires the same word, and the reads after it see what the earlier
// releasers wrote
__device__ __forceinline__ int atomic_add_acq_rel(int* ptr, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(ptr), "r"(v) : "memory");
  return old;
}

template <typename T>
__global__ void __launch_bounds__(kUnmaskThreads) unmask_kernel(const UnmaskParams p) {
  using VT = VecTraits<T>;
  constexpr int N = VT::kN;
  pdl_trigger();
  pdl_wait();
  if (skip_requested(p.skip_if)) {
    // a step after the block completed: nothing to do; the done word stays raised
    if (blockIdx.x == 0 && threadIdx.x == 0 && p.all_done) *p.all_done = 1;
    return;
  }
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
  // each thread's own ring of kUnmaskRing vectors (slot-major: consecutive threads, consecutive 16 B)
  __shared__ __align__(16) uint4 s_ring[kUnmaskRing][kUnmaskThreads];
  __shared__ int s_flag;
  const int warp = tid >> 5, lane = tid & 31;

  // A row's part of the range is a segment. Each thread streams its vectors of the segment
  // through its own ring, starting at slot 0; the first kUnmaskRing copies of a segment are
  // issued here, for the next segment before the CTA reduces the finished one, so that those
  // loads are in flight during the reduction.
  auto prologue = [&](long long sg) {
    const int rw = (int)(sg / p.vec_per_row);
    const long long rb = (long long)rw * p.vec_per_row;
    const long long se = min(vend, rb + p.vec_per_row);
    const int n = (se - sg > tid) ? (int)((se - sg - tid + kUnmaskThreads - 1) / kUnmaskThreads) : 0;
    const uint4* src = base + sg + tid;
#pragma unroll
    for (int i = 0; i < kUnmaskRing; ++i) {
      if (i < n) cp_async16(&s_ring[i][tid], src + i * kUnmaskThreads);
      cp_async_commit();
    }
  };
  if (vbeg < vend) prologue(vbeg);

  for (long long seg = vbeg; seg < vend;) {
    const int row = (int)(seg / p.vec_per_row);
    const long long row_beg = (long long)row * p.vec_per_row;
    const long long seg_end = min(vend, row_beg + p.vec_per_row);
    const int vb = (int)(seg - row_beg), ve = (int)(seg_end - row_beg);   // vectors of this row
    const uint4* vp = base + row_beg;

    // running state: m, the lowest index attaining it, and sum 2^(c (x - m)) kept as two packed
    // pairs of partial sums (four independent accumulation chains)
    float m = -INFINITY;
    int32_t idx = 0x7fffffff;
    const uint64_t c2 = pack_f32x2(c, c);
    uint64_t nmc2 = pack_f32x2(0.f, 0.f);
    uint64_t acc[2] = {pack_f32x2(0.f, 0.f), pack_f32x2(0.f, 0.f)};
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
      float vm;
      if constexpr (N == 8) {
        vm = fmax3(fmax3(x[0], x[1], x[2]), fmax3(x[3], x[4], x[5]), fmaxf(x[6], x[7]));
      } else {
        vm = fmax3(x[0], x[1], fmaxf(x[2], x[3]));
      }
      if (vm > m) {
        // a new running maximum (rare once a row's first vectors have been seen): its lowest
        // index in this vector, and the partial sums moved to the new base
        int vi = N - 1;
#pragma unroll
        for (int k = N - 1; k >= 0; --k)
          if (x[k] == vm) vi = k;
        const float f = (m == -INFINITY) ? 0.f : ex2(c * (m - vm));
        const uint64_t f2 = pack_f32x2(f, f);
        acc[0] = fmul_f32x2(acc[0], f2);
        acc[1] = fmul_f32x2(acc[1], f2);
        m = vm;
        idx = vbase + vi;
        nmc2 = pack_f32x2(-c * m, -c * m);
      }
#pragma unroll
      for (int k = 0; k < N / 2; ++k) {
        const uint64_t e2 = ffma_f32x2(pack_f32x2(x[2 * k], x[2 * k + 1]), c2, nmc2);
        acc[k & 1] = fadd_f32x2(acc[k & 1], pack_f32x2(ex2(lo_f32(e2)), ex2(hi_f32(e2))));
      }
    };
    // this thread's vectors vb + tid + i * kUnmaskThreads, i < nv, stream through its ring: the
    // copy of vector i + kUnmaskRing is issued once vector i has been consumed, so kUnmaskRing
    // copies stay in flight (one commit group per index, empty past the end, keeps the count);
    // copies 0 .. kUnmaskRing - 1 were issued by prologue()
    const int nv = (ve - vb > tid) ? (ve - vb - tid + kUnmaskThreads - 1) / kUnmaskThreads : 0;
    auto issue = [&](int i) {
      if (i < nv) cp_async16(&s_ring[i % kUnmaskRing][tid], vp + vb + tid + i * kUnmaskThreads);
      cp_async_commit();
    };
    for (int i = 0; i < nv; ++i) {
      cp_async_wait<kUnmaskRing - 1>();   // the oldest copy (vector i) has landed
      const uint4 raw = s_ring[i % kUnmaskRing][tid];
      consume(raw, vb + tid + i * kUnmaskThreads);
      issue(i + kUnmaskRing);
    }
    cp_async_wait<0>();
    if (seg_end < vend) prologue(seg_end);

    // ---- CTA reduction (warp shuffles, then across warps), lowest index on ties
    const uint64_t accs = fadd_f32x2(acc[0], acc[1]);
    RedState st{m, lo_f32(accs) + hi_f32(accs), idx};
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
        // the ticket releases this CTA's partial and acquires those of the CTAs counted before it
        const int old = atomic_add_acq_rel(row_cnt + row, 1);
        row_done = (old == (int)(c_hi - c_lo));
        if (row_done) {
          row_cnt[row] = 0;
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
        // releases this row's confidence and argmax; the sequence's last row acquires the others'
        // (the CTA barrier below passes them on to the threads of commit_sequence)
        const int b = row / p.block_size;
        const int old = atomic_add_acq_rel(seq_cnt + b, 1);
        if (old == p.block_size - 1) {
          seq_cnt[b] = 0;
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
  L.done = take(sizeof(unsigned long long));
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
  p.keep_masked = predict_noise_keep(a->block_size, a->keep_masked, a->noise_steps, a->noise_step);
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
  p.batch = a->batch;
  p.off_done = pl.layout.done;
  p.skip_if = a->skip_if;
  p.all_done = a->all_done;
  if (a->dtype == TT_BF16)
    launch_pdl(unmask_kernel<__nv_bfloat16>, dim3(pl.grid), dim3(kUnmaskThreads), 0, stream, p);
  else
    launch_pdl(unmask_kernel<float>, dim3(pl.grid), dim3(kUnmaskThreads), 0, stream, p);
  return cudaGetLastError() == cudaSuccess ? TT_OK : TT_ERR_CUDA;
}

// ---------------------------------------------------------------- fused LM head + unmask
// The same step from the hidden states instead of the logits: logits = x W^T (x [B*S][D] the
// final hidden states, W [V][D] the LM-head weight) are formed tile by tile on the tensor cores
// and reduced to (max, sum exp, argmax) in the epilogue, so the [B*S][V] logits never reach
// memory. A CTA owns one 128-row tile of x (M tile) and a contiguous range of 128-column
// vocabulary tiles; per vocabulary tile it runs the K loop over D in 64-wide stages (both
// operands K-major, 128B-swizzled, brought in by TMA without multicast) into one of two TMEM
// accumulators, while its epilogue warps reduce the other. The per-range partial states of a row
// are merged by the last CTA of the M tile to finish (ticket), which then applies the commit rule
// (either sampler) to every sequence whose rows are all merged.
namespace {

constexpr int kLmThreads = 192;                       // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kLmStages = 6;
constexpr uint32_t kLmBox = 128 * 128;                // 128 rows x 64 bf16 = 16 KB
constexpr uint32_t kLmStageBytes = 2 * kLmBox;        // x box + W box
constexpr uint32_t kLmTiles = kLmStages * kLmStageBytes;   // 192 KB
constexpr uint32_t kLmSmem = kLmTiles + 2048 + 1024;  // barriers / lists + alignment slack
constexpr uint32_t kLmTmemCols = 256;                 // two 128-column accumulators
constexpr uint32_t kLmIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(128 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);

struct LmParams {
  CUtensorMap tm_x, tm_w;
  UnmaskParams u;                 // commit rule, outputs, workspace offsets of conf / argmax / sequence tickets
  int32_t M, D, V, nvr, vtiles;
  size_t off_parts, off_mt_cnt;
};

struct LmSmem {
  uint64_t full[kLmStages], empty[kLmStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int last_flag;
  int n_commit;
  int commit_list[128];
};

__device__ __forceinline__ uint64_t lm_sdesc(uint32_t saddr) {
  // K-major, 128B swizzle: 8-row groups 1024 bytes apart
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) |
         ((uint64_t)2 << 61);
}

__global__ void __launch_bounds__(kLmThreads, 1) lmhead_unmask_kernel(const __grid_constant__ LmParams p) {
  extern __shared__ __align__(1024) uint8_t lm_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(lm_raw) + 1023) & ~uintptr_t(1023));
  LmSmem& sm = *reinterpret_cast<LmSmem*>(tiles + kLmTiles);
  const UnmaskParams& u = p.u;
  WsHeader* hdr = reinterpret_cast<WsHeader*>(u.ws);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int mt = blockIdx.x / p.nvr, vr = blockIdx.x % p.nvr;
  const int t0 = (int)((long long)vr * p.vtiles / p.nvr), t1 = (int)((long long)(vr + 1) * p.vtiles / p.nvr);
  const int ntile = t1 - t0, nk = p.D / 64;
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < kLmStages; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.acc_full[i], 1);
      mbar_init(&sm.acc_empty[i], 128);
    }
    mbar_init(&sm.drain, 1);
    fence_barrier_init();
    prefetch_tmap(&p.tm_x);
    prefetch_tmap(&p.tm_w);
    sm.abort_flag = 0;
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kLmTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  pdl_trigger();
  pdl_wait();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (skip_requested(u.skip_if)) {
    // a step after the block completed: release TMEM and leave; the done word stays raised
    if (warp == 1) tmem_dealloc(tmem, kLmTmemCols);
    if (blockIdx.x == 0 && tid == 0 && u.all_done) *u.all_done = 1;
    return;
  }
  volatile int* abort_flag = &sm.abort_flag;
  auto fail = [&](uint32_t detail) {
    report_error(hdr, TT_ERR_DEVICE_TIMEOUT, detail);
    *abort_flag = 1;
  };
  const uint32_t tiles_s = smem_u32(tiles);

  if (warp == 0) {
    // ======================= TMA producer: (x box, W box) per 64-wide K step
    if (lane == 0) {
      long long it = 0;
      bool ok = true;
      for (int n = 0; n < ntile && ok; ++n) {
        for (int ks = 0; ks < nk; ++ks, ++it) {
          const int stage = (int)(it % kLmStages);
          const uint32_t round = (uint32_t)(it / kLmStages);
          if (round > 0 && !mbar_wait_bounded(&sm.empty[stage], (round - 1) & 1, abort_flag)) {
            fail(kDetailWaitKvEmpty);
            ok = false;
            break;
          }
          uint8_t* dst = tiles + stage * kLmStageBytes;
          mbar_arrive_expect_tx(&sm.full[stage], kLmStageBytes);
          tma_load_3d(dst, &p.tm_x, &sm.full[stage], ks * 64, 0, mt * 128);
          tma_load_3d(dst + kLmBox, &p.tm_w, &sm.full[stage], ks * 64, 0, (t0 + n) * 128);
        }
      }
      for (long long j = (it > kLmStages ? it - kLmStages : 0); j < it; ++j) {
        const uint64_t tw = globaltimer_ns();
        while (!mbar_try_wait(&sm.full[j % kLmStages], (uint32_t)((j / kLmStages) & 1)) &&
               globaltimer_ns() - tw < kWaitLimitNs) {
        }
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer: acc[n % 2] = x_tile W_tile^T over D
    if (lane == 0) {
      long long it = 0;
      bool ok = true;
      for (int n = 0; n < ntile && ok; ++n) {
        const int acc = n & 1;
        if (n >= 2 && !mbar_wait_bounded(&sm.acc_empty[acc], (uint32_t)(((n - 2) >> 1) & 1), abort_flag)) {
          fail(kDetailWaitPvDone);
          break;
        }
        tc_fence_after();
        const uint32_t d_tm = tmem + 128u * (uint32_t)acc;
        for (int ks = 0; ks < nk; ++ks, ++it) {
          const int stage = (int)(it % kLmStages);
          if (!mbar_wait_bounded(&sm.full[stage], (uint32_t)((it / kLmStages) & 1), abort_flag)) {
            fail(kDetailWaitKvFull);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t da = lm_sdesc(tiles_s + stage * kLmStageBytes);
          const uint64_t db = lm_sdesc(tiles_s + stage * kLmStageBytes + kLmBox);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(d_tm, da + (uint64_t)((kk * 32) >> 4), db + (uint64_t)((kk * 32) >> 4), kLmIdesc,
                   (ks > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&sm.empty[stage]);
        }
        if (ok) tc_commit(&sm.acc_full[acc]);
      }
    }
  } else {
    // ======================= epilogue: thread = row (TMEM lane), running (max, sum exp, argmax)
    const int r = 32 * (warp & 3) + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float c = u.c;
    float m = -INFINITY, s = 0.f;
    int32_t idx = 0x7fffffff;
    for (int n = 0; n < ntile; ++n) {
      const int acc = n & 1;
      if (!mbar_wait_bounded(&sm.acc_full[acc], (uint32_t)((n >> 1) & 1), abort_flag)) {
        fail(kDetailWaitSFull);
        break;
      }
      __syncwarp();
      tc_fence_after();
      uint32_t v[128];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        tmem_ld32(tmem + lane_off + 128u * (uint32_t)acc + 32u * (uint32_t)q, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * q]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&sm.acc_empty[acc]);   // the accumulator can take tile n + 2
      const int vbase = (t0 + n) * 128;
      if (u.exclude_mask_token) {
        const int e = u.mask_token_id - vbase;
#pragma unroll
        for (int j = 0; j < 128; ++j)   // static indices keep v[] in registers
          if (j == e) v[j] = __float_as_uint(-INFINITY);
      }
      float tmax = __uint_as_float(v[0]);
      int targ = 0;
#pragma unroll
      for (int j = 1; j < 128; ++j) {
        if (__uint_as_float(v[j]) > tmax) {
          tmax = __uint_as_float(v[j]);
          targ = j;
        }
      }
      const float nm = fmaxf(m, tmax);
      float ts = 0.f;
#pragma unroll
      for (int j = 0; j < 128; ++j) ts += ex2(c * (__uint_as_float(v[j]) - nm));
      s = ((m == -INFINITY) ? 0.f : s * ex2(c * (m - nm))) + ts;
      if (tmax > m) idx = vbase + targ;   // strictly larger: an earlier tile keeps ties
      m = nm;
    }
    UnmaskPartial* parts = reinterpret_cast<UnmaskPartial*>(u.ws + p.off_parts);
    parts[((size_t)mt * p.nvr + vr) * 128 + r] = UnmaskPartial{m, s, idx, 0};
  }

  // ---- teardown of the tile phase: MMAs drained, TMEM released
  if (warp == 1 && lane == 0) {
    tc_commit(&sm.drain);
    const uint64_t tw = globaltimer_ns();
    while (!mbar_try_wait(&sm.drain, 0) && globaltimer_ns() - tw < kWaitLimitNs) {
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kLmTmemCols);
  }
  if (*abort_flag) return;   // uniform: read after the barrier

  // ---- the last CTA of this M tile merges its rows' partial states and commits finished sequences
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    int* mt_cnt = reinterpret_cast<int*>(u.ws + p.off_mt_cnt);
    const int old = atomicAdd(mt_cnt + mt, 1);
    sm.last_flag = (old == p.nvr - 1) ? 1 : 0;
    if (sm.last_flag) mt_cnt[mt] = 0;
    sm.n_commit = 0;
  }
  __syncthreads();
  if (!sm.last_flag) return;
  __threadfence();
  float* conf_ws = reinterpret_cast<float*>(u.ws + u.off_conf);
  int32_t* arg_ws = reinterpret_cast<int32_t*>(u.ws + u.off_argmax);
  int* seq_cnt = reinterpret_cast<int*>(u.ws + u.off_seq_cnt);
  const float4* pp = reinterpret_cast<const float4*>(u.ws + p.off_parts);
  if (tid < 128) {
    const int row = mt * 128 + tid;
    if (row < p.M) {
      // the row's nvr partial states, loaded 16 at a time (independent loads in flight) and
      // combined in range order, so ties still resolve to the lowest token id
      const float4* base = pp + (size_t)mt * p.nvr * 128 + tid;
      RedState st{-INFINITY, 0.f, 0x7fffffff};
      for (int k0 = 0; k0 < p.nvr; k0 += 16) {
        float4 q[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (k0 + j < p.nvr) q[j] = __ldcg(base + (size_t)(k0 + j) * 128);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (k0 + j < p.nvr) st = red_combine(st, RedState{q[j].x, q[j].y, __float_as_int(q[j].z)}, u.c);
      }
      const float conf = 1.0f / st.s;
      conf_ws[row] = conf;
      arg_ws[row] = st.idx;
      if (u.conf_out) u.conf_out[row] = conf;
      if (u.argmax_out) u.argmax_out[row] = st.idx;
      __threadfence();
      const int b = row / u.block_size;
      const int old = atomicAdd(seq_cnt + b, 1);
      if (old == u.block_size - 1) {
        seq_cnt[b] = 0;
        __threadfence();
        sm.commit_list[atomicAdd(&sm.n_commit, 1)] = b;
      }
    }
  }
  __syncthreads();
  const int nc = sm.n_commit;
  for (int i = 0; i < nc; ++i) {
    commit_sequence(u, sm.commit_list[i], conf_ws, arg_ws);
    __syncthreads();   // commit_sequence reuses its shared counters
  }
}

// 3-D bf16 map (D [contiguous], 1, rows), box (64, 1, 128), 128B swizzle.
bool lm_make_map(CUtensorMap* m, const void* base, int D, long long rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  const cuuint64_t dims[3] = {(cuuint64_t)D, 1, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)D * 2};
  const cuuint32_t box[3] = {64, 1, 128};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct LmLayout {
  int n_mt, nvr;
  size_t parts, mt_cnt, seq_cnt, done, conf, argmax, total;
};

LmLayout lm_layout(const tt_lmhead_unmask_args_t* a, int num_sms) {
  LmLayout L{};
  const int M = a->batch * a->block_size;
  L.n_mt = (M + 127) / 128;
  L.nvr = std::max(1, std::min(a->vocab / 128, std::max(1, num_sms) / L.n_mt));
  size_t off = kHeaderBytes;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = (off + bytes + 255) & ~size_t(255);
    return o;
  };
  L.parts = take(sizeof(UnmaskPartial) * (size_t)L.n_mt * L.nvr * 128);
  L.mt_cnt = take(sizeof(int) * (size_t)L.n_mt);
  L.seq_cnt = take(sizeof(int) * (size_t)a->batch);
  L.done = take(sizeof(unsigned long long));
  L.conf = take(sizeof(float) * (size_t)M);
  L.argmax = take(sizeof(int32_t) * (size_t)M);
  L.total = off;
  return L;
}

}  // namespace

size_t lmhead_workspace_bytes(const tt_lmhead_unmask_args_t* a, int num_sms) { return lm_layout(a, num_sms).total; }

int lmhead_unmask_launch(const tt_lmhead_unmask_args_t* a, void* ws, cudaStream_t stream) {
  const LmLayout L = lm_layout(a, device_sm_count());
  LmParams p{};
  const int M = a->batch * a->block_size;
  if (!lm_make_map(&p.tm_x, a->x, a->hidden, M)) return TT_ERR_CUDA;
  if (!lm_make_map(&p.tm_w, a->w, a->hidden, a->vocab)) return TT_ERR_CUDA;
  UnmaskParams& u = p.u;
  u.block_size = a->block_size;
  u.rows = M;
  u.c = a->inv_temperature * 1.4426950408889634f;
  u.gamma = a->gamma;
  u.mask_token_id = a->mask_token_id;
  u.exclude_mask_token = a->exclude_mask_token;
  u.remaining_steps = a->remaining_steps;
  u.sampler = a->sampler;
  u.keep_masked = predict_noise_keep(a->block_size, a->keep_masked, a->noise_steps, a->noise_step);
  u.tokens = a->tokens;
  u.is_masked = a->is_masked;
  u.conf_out = a->conf;
  u.argmax_out = a->argmax;
  u.n_committed = a->n_committed;
  u.n_masked = a->n_masked;
  u.ws = static_cast<uint8_t*>(ws);
  u.off_seq_cnt = L.seq_cnt;
  u.off_conf = L.conf;
  u.off_argmax = L.argmax;
  u.batch = a->batch;
  u.off_done = L.done;
  u.skip_if = a->skip_if;
  u.all_done = a->all_done;
  p.M = M;
  p.D = a->hidden;
  p.V = a->vocab;
  p.nvr = L.nvr;
  p.vtiles = a->vocab / 128;
  p.off_parts = L.parts;
  p.off_mt_cnt = L.mt_cnt;
  static unsigned long long attr_done = 0;   // bit per device ordinal (< 64)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TT_ERR_CUDA;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(__atomic_load_n(&attr_done, __ATOMIC_ACQUIRE) & bit)) {
    if (cudaFuncSetAttribute(lmhead_unmask_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kLmSmem) !=
        cudaSuccess)
      return TT_ERR_CUDA;
    __atomic_fetch_or(&attr_done, bit, __ATOMIC_ACQ_REL);
  }
  return launch_pdl(lmhead_unmask_kernel, dim3(L.n_mt * L.nvr), dim3(kLmThreads), kLmSmem, stream, p) == cudaSuccess
             ? TT_OK
             : TT_ERR_CUDA;
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
// Per device: the context whose copy of the scratch was last set up, and its address. A context
// that is destroyed and created again (cudaDeviceReset, or a runtime that tears down the primary
// context) loads this module afresh, so the symbol may move: the set-up runs again whenever the
// current context or the looked-up address differs from the recorded one.
void* g_static_ctx[kMaxDevices] = {};
uint8_t* g_static_ptr[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
  }
  return fn;
}
}  // namespace

int unmask_launch_static(const tt_unmask_args_t* a, cudaStream_t stream) {
  const long long rows = (long long)a->batch * a->block_size;
  if (rows > kStaticMaxRows) return TT_ERR_WORKSPACE_TOO_SMALL;
  const UnmaskLayout L = layout_for(kStaticMaxRows, kStaticMaxRows, kStaticMaxGrid);
  if (L.total > kStaticScratchBytes) return TT_ERR_WORKSPACE_TOO_SMALL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TT_ERR_CUDA;
  // The array's device address, looked up on every call: a host-side table lookup that allocates
  // nothing (the host-side name g_unmask_scratch is only a stand-in, never a device address).
  // The lookup also initialises the runtime's context for this device if nothing has yet.
  void* sym = nullptr;
  if (cudaGetSymbolAddress(&sym, g_unmask_scratch) != cudaSuccess || !sym) return TT_ERR_CUDA;
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  CUcontext ctx = nullptr;
  if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return TT_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(sym);
  {
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (g_static_ctx[dev] != static_cast<void*>(ctx) || g_static_ptr[dev] != ws) {
      // Set-up, once per device and context, with that device current: clear the header and
      // the ticket counters (everything before the partial slots), stream-ordered before the
      // first launch. (A freshly loaded module holds zeros already; the clearing makes the state
      // explicit rather than relying on it.)
      if (cudaMemsetAsync(ws, 0, L.partials, stream) != cudaSuccess) return TT_ERR_CUDA;
      g_static_ptr[dev] = ws;
      g_static_ctx[dev] = static_cast<void*>(ctx);
    }
  }
  UnmaskPlan pl = unmask_plan(a, device_sm_count());
  pl.grid = std::min(pl.grid, kStaticMaxGrid);
  pl.layout = L;
  return unmask_launch(a, pl, ws, stream);
}

// ---------------------------------------------------------------- Algorithm 2: the time input
// tau_b = |{l : position l of sequence b is masked}| / S, one warp per sequence, so a multi-step
// refinement loop can feed the next step's time input from the mask on the device.
constexpr int kTauThreads = 128;

__global__ void __launch_bounds__(kTauThreads) block_tau_kernel(const uint8_t* __restrict__ is_masked, int B, int S,
                                                                float* __restrict__ tau, const int32_t* skip_if) {
  pdl_trigger();
  pdl_wait();
  if (skip_requested(skip_if)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x * (kTauThreads / 32) + warp;
  if (b >= B) return;
  int n = 0;
  for (int l = lane; l < S; l += 32) n += is_masked[(size_t)b * S + l] ? 1 : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
  if (lane == 0) tau[b] = (float)n / (float)S;
}

int block_tau_launch(const uint8_t* is_masked, int B, int S, float* tau, const int32_t* skip_if,
                     cudaStream_t stream) {
  const int per = kTauThreads / 32;
  return launch_pdl(block_tau_kernel, dim3((B + per - 1) / per), dim3(kTauThreads), 0, stream, is_masked, B, S, tau,
                    skip_if) ==
                 cudaSuccess
             ? TT_OK
             : TT_ERR_CUDA;
}

}  // namespace tt
