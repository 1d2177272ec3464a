// Eq. (1) of "Nemotron-TwoTower: Diffusion Language Modeling with Pretrained AR Context" (§2.1,
// "Bidirectional attention") for fp32 tensors on the sm_100a tensor cores (tcgen05.mma kind::tf32).
//
// fp32 inputs carry an absolute 1e-5 accuracy bar. One tf32 product keeps 11 significant bits, so
// each operand is split into a tf32 head and an fp32 tail, x = x_hi + x_lo with x_hi = x with its
// low 13 mantissa bits cleared (exact in tf32) and x_lo = x - x_hi (exact in fp32, |x_lo| < 2^-10 |x|),
// and every product is formed as a_hi b_hi + a_hi b_lo + a_lo b_hi on the tensor cores with fp32
// accumulation; the dropped a_lo b_lo term and the tf32 rounding of the tails are near 2^-21 of
// the product, far below the bar (the three-product split of one fp32 product, as in 3xTF32).
//
// One CTA of 128 threads per 128-row query tile of a group (sequence b, kv head): rows
// m = s * G + g as in the bf16 path, one thread per row (its TMEM lane). Keys stream in tiles of
// 32 (context tokens through the page table or the contiguous slab, then the block's S tokens).
// Per tile the threads load K and V with coalesced plain loads, split them and write K_hi / K_lo
// (K-major) and V^T_hi / V^T_lo (V transposed, so the PV product's B operand is K-major too) in
// the 128-byte-swizzled layout the MMA descriptors read; thread 0 issues S = Q K^T (three
// products per 8-wide K step); the threads load their score row from TMEM, run the online
// softmax in fp32 (exp2 with the scale folded in, exact rescaling of O when the maximum moves),
// write P_hi and P_lo to TMEM, and thread 0 issues O += P V (A = P from TMEM). The fp32 workloads
// are small, so the tile steps run one after the other and no split-KV is needed.
#include <cmath>

#include "tt_common.cuh"
#include "tt_internal.h"

namespace tt {

namespace {

constexpr int kTfThreads = 128;
constexpr int kTfRows = 128;     // query rows per CTA (one M=128 MMA)
constexpr int kTfKeys = 32;      // keys per tile (one 128-byte swizzle row of fp32)
constexpr uint32_t kTfTmemCols = 256;
// TMEM columns: O [0, D), S and then P_hi [128, 160), P_lo [160, 192)
constexpr uint32_t kTmS = 128, kTmPlo = 160;

struct Tf32Params {
  const float* q;
  const float* k_blk;
  const float* v_blk;
  const float* k_ctx;
  const float* v_ctx;
  const int32_t* ctx_lens;
  const int32_t* page_table;
  int32_t B, S, Hq, Hkv, G;
  int32_t page_size, max_pages, num_pages, ctx_stride;
  float scale_log2;   // softmax_scale * log2(e)
  float* out;
  float* lse;
  WsHeader* hdr;
  const int32_t* skip_if;
};

// Instruction descriptor, kind::tf32: D fp32, A and B tf32, both K-major.
constexpr uint32_t tf32_idesc(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_ss_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_ts_tf32(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Shared-memory descriptor of a K-major operand in 128-byte swizzle atoms (8-row groups 1024 B apart).
__device__ __forceinline__ uint64_t tf_sdesc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) |
         ((uint64_t)2 << 61);
}

// Byte offset of element (r, k), k < 32, in a K-major atom of rows x 32 fp32 with 128-byte
// swizzle: rows of 128 bytes, the 16-byte chunk index XORed with the row index mod 8.
__device__ __forceinline__ uint32_t sw128_f32(int r, int k) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((((k >> 2) ^ r) & 7) << 4) + (k & 3) * 4);
}

__device__ __forceinline__ float tf32_head(float x) { return __uint_as_float(__float_as_uint(x) & 0xffffe000u); }

template <int D>
struct TfLayout {
  static constexpr uint32_t kQ = kTfRows * D * 4;          // Q_hi (and Q_lo), D/32 atoms of 128 rows
  static constexpr uint32_t kK = kTfKeys * D * 4;          // K_hi (and K_lo), D/32 atoms of 32 rows
  static constexpr uint32_t kV = D * kTfKeys * 4;          // V^T_hi (and V^T_lo), one atom of D rows
  static constexpr uint32_t kQhi = 0, kQlo = kQ, kKhi = 2 * kQ, kKlo = kKhi + kK, kVhi = kKlo + kK, kVlo = kVhi + kV;
  static constexpr uint32_t kBar = kVlo + kV;
  static constexpr uint32_t kBytes = kBar + 256 + 1024;   // barriers + alignment slack
};

template <int D>
__global__ void __launch_bounds__(kTfThreads, 1) attn_tf32_kernel(const Tf32Params p) {
  using L = TfLayout<D>;
  extern __shared__ __align__(1024) uint8_t tf_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tf_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar_s = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* bar_o = bar_s + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_s + 2);
  int* abort_flag = reinterpret_cast<int*>(bar_s + 3);
  const int t = threadIdx.x, warp = t >> 5;
  const int b = blockIdx.z, kvh = blockIdx.y, row0 = blockIdx.x * kTfRows;
  const int M = p.G * p.S;

  if (t == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTfTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  pdl_trigger();
  pdl_wait();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  if (skip_requested(p.skip_if)) {
    if (warp == 0) tmem_dealloc(tmem, kTfTmemCols);
    return;
  }

  int L_b = p.ctx_lens[b];
  if (L_b < 0) {
    if (t == 0) report_error(p.hdr, TT_ERR_DEVICE, kDetailNegativeLen);
    L_b = 0;
  }
  const int cap = p.page_table ? p.max_pages * p.page_size : p.ctx_stride;
  if (L_b > cap) {
    if (t == 0) report_error(p.hdr, TT_ERR_DEVICE, kDetailCtxTooLong);
    L_b = cap;
  }
  const int n_keys = L_b + p.S;

  // ---- this CTA's query rows, split and swizzled (rows past M are zero)
  for (int e = t; e < kTfRows * D; e += kTfThreads) {
    const int r = e / D, c = e - r * D;
    const int m = row0 + r;
    float x = 0.f;
    if (m < M) {
      const int s = m / p.G, g = m - s * p.G;
      x = p.q[(((size_t)b * p.S + s) * p.Hq + kvh * p.G + g) * D + c];
    }
    const float hi = tf32_head(x);
    const uint32_t off = (uint32_t)(c >> 5) * (kTfRows * 128) + sw128_f32(r, c & 31);
    *reinterpret_cast<float*>(smem + L::kQhi + off) = hi;
    *reinterpret_cast<float*>(smem + L::kQlo + off) = x - hi;
  }

  const uint32_t s_base = smem_u32(smem);
  const uint32_t idesc_qk = tf32_idesc(kTfRows, kTfKeys);
  const uint32_t idesc_pv = tf32_idesc(kTfRows, D);
  const float sc = p.scale_log2;
  float m_run = -INFINITY, l_run = 0.f;
  const int n_tiles = (n_keys + kTfKeys - 1) / kTfKeys;
  bool ok = true;
  uint32_t o_commits = 0;   // bar_o phases thread 0 has committed
  for (int j = 0; j < n_tiles && ok; ++j) {
    const int key0 = j * kTfKeys;
    // ---- K and V rows of this tile: split, K-major K, transposed V (keys past the end are zero)
    for (int e = t; e < kTfKeys * D; e += kTfThreads) {
      const int kr = e / D, c = e - kr * D;
      const int key = key0 + kr;
      float kx = 0.f, vx = 0.f;
      if (key < L_b) {
        size_t row;
        if (p.page_table) {
          int pg = p.page_table[(size_t)b * p.max_pages + key / p.page_size];
          if (pg < 0 || pg >= p.num_pages) {
            report_error(p.hdr, TT_ERR_DEVICE, kDetailBadPage);
            pg = 0;   // read a valid page instead; the result is unspecified, the error is set
          }
          row = (size_t)pg * p.page_size + key % p.page_size;
        } else {
          row = (size_t)b * p.ctx_stride + key;
        }
        const size_t idx = (row * p.Hkv + kvh) * D + c;
        kx = p.k_ctx[idx];
        vx = p.v_ctx[idx];
      } else if (key < n_keys) {
        const size_t idx = (((size_t)b * p.S + (key - L_b)) * p.Hkv + kvh) * D + c;
        kx = p.k_blk[idx];
        vx = p.v_blk[idx];
      }
      const float khi = tf32_head(kx), vhi = tf32_head(vx);
      const uint32_t koff = (uint32_t)(c >> 5) * (kTfKeys * 128) + sw128_f32(kr, c & 31);
      *reinterpret_cast<float*>(smem + L::kKhi + koff) = khi;
      *reinterpret_cast<float*>(smem + L::kKlo + koff) = kx - khi;
      const uint32_t voff = sw128_f32(c, kr);
      *reinterpret_cast<float*>(smem + L::kVhi + voff) = vhi;
      *reinterpret_cast<float*>(smem + L::kVlo + voff) = vx - vhi;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // generic writes -> tensor-core reads
    __syncthreads();
    // ---- S = Q K^T: per 8-wide K step, Q_hi K_hi + Q_hi K_lo + Q_lo K_hi
    if (t == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 8; ++kk) {
        const uint32_t qo = (uint32_t)((kk >> 2) * (kTfRows * 128) + (kk & 3) * 32);
        const uint32_t ko = (uint32_t)((kk >> 2) * (kTfKeys * 128) + (kk & 3) * 32);
        const uint64_t qh = tf_sdesc(s_base + L::kQhi + qo), ql = tf_sdesc(s_base + L::kQlo + qo);
        const uint64_t kh = tf_sdesc(s_base + L::kKhi + ko), kl = tf_sdesc(s_base + L::kKlo + ko);
        mma_ss_tf32(tmem + kTmS, qh, kh, idesc_qk, kk > 0 ? 1u : 0u);
        mma_ss_tf32(tmem + kTmS, qh, kl, idesc_qk, 1u);
        mma_ss_tf32(tmem + kTmS, ql, kh, idesc_qk, 1u);
      }
      tc_commit(bar_s);
    }
    bool failed = !mbar_wait_bounded(bar_s, (uint32_t)(j & 1), abort_flag);
    if (__syncthreads_or(failed)) {
      if (t == 0) report_error(p.hdr, TT_ERR_DEVICE_TIMEOUT, kDetailWaitSFull);
      ok = false;
      break;
    }
    tc_fence_after();
    // ---- online softmax on this thread's row
    uint32_t sr[32];
    tmem_ld32(tmem + lane_off + kTmS, sr);
    tmem_wait_ld();
    float mt = -INFINITY;
#pragma unroll
    for (int c = 0; c < kTfKeys; ++c) {
      if (key0 + c >= n_keys) sr[c] = __float_as_uint(-INFINITY);
      mt = fmaxf(mt, __uint_as_float(sr[c]) * sc);
    }
    const float m_new = fmaxf(m_run, mt);
    const float factor = (m_run == -INFINITY) ? 0.f : ex2(m_run - m_new);
    uint32_t phi[32], plo[32];
    float psum = 0.f;
#pragma unroll
    for (int c = 0; c < kTfKeys; ++c) {
      const float pv = ex2(fmaf(__uint_as_float(sr[c]), sc, -m_new));
      psum += pv;
      const float h = tf32_head(pv);
      phi[c] = __float_as_uint(h);
      plo[c] = __float_as_uint(pv - h);
    }
    l_run = l_run * factor + psum;
    m_run = m_new;
    tmem_st32(tmem + lane_off + kTmS, phi);
    tmem_st32(tmem + lane_off + kTmPlo, plo);
    if (j > 0 && __any_sync(0xffffffffu, factor != 1.0f)) {
      // exact rescale of the running output (the PV of the previous tile has completed)
#pragma unroll 1
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t orr[32];
        tmem_ld32(tmem + lane_off + 32u * (uint32_t)cb, orr);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * factor);
        tmem_st32(tmem + lane_off + 32u * (uint32_t)cb, orr);
      }
    }
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();
    // ---- O += P V: per 8-wide K step, P_hi V_hi + P_hi V_lo + P_lo V_hi
    if (t == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < kTfKeys / 8; ++kk) {
        const uint64_t vh = tf_sdesc(s_base + L::kVhi + kk * 32), vl = tf_sdesc(s_base + L::kVlo + kk * 32);
        mma_ts_tf32(tmem, tmem + kTmS + 8u * (uint32_t)kk, vh, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        mma_ts_tf32(tmem, tmem + kTmS + 8u * (uint32_t)kk, vl, idesc_pv, 1u);
        mma_ts_tf32(tmem, tmem + kTmPlo + 8u * (uint32_t)kk, vh, idesc_pv, 1u);
      }
      tc_commit(bar_o);
      ++o_commits;
    }
    // the PV product reads this tile's shared memory and P: it completes before either is reused
    failed = !mbar_wait_bounded(bar_o, (uint32_t)(j & 1), abort_flag);
    if (__syncthreads_or(failed)) {
      if (t == 0) report_error(p.hdr, TT_ERR_DEVICE_TIMEOUT, kDetailWaitPvDone);
      ok = false;
      break;
    }
    tc_fence_after();
  }

  if (ok) {
    // ---- epilogue: O / l for this thread's row, and the natural-log log-sum-exp
    const int m = row0 + t;
    const bool valid = m < M;
    const int s = valid ? m / p.G : 0, g = valid ? m - s * p.G : 0;
    const int h = kvh * p.G + g;
    const float inv = 1.0f / l_run;
    float* dst = p.out + (((size_t)b * p.S + s) * p.Hq + h) * D;
#pragma unroll 1
    for (int cb = 0; cb < D / 32; ++cb) {
      uint32_t orr[32];
      tmem_ld32(tmem + lane_off + 32u * (uint32_t)cb, orr);
      tmem_wait_ld();
      if (valid) {
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4)
          reinterpret_cast<float4*>(dst + 32 * cb)[q4] =
              make_float4(__uint_as_float(orr[4 * q4]) * inv, __uint_as_float(orr[4 * q4 + 1]) * inv,
                          __uint_as_float(orr[4 * q4 + 2]) * inv, __uint_as_float(orr[4 * q4 + 3]) * inv);
      }
    }
    if (valid && p.lse) p.lse[((size_t)b * p.Hq + h) * p.S + s] = (m_run + log2f(l_run)) * 0.69314718055994531f;
  }
  // ---- teardown: every MMA has completed (each tile waited for its PV; an abort drains here:
  // one more commit on bar_o completes its next phase once everything issued before it has)
  if (t == 0) {
    tc_commit(bar_o);
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar_o, o_commits & 1u) && globaltimer_ns() - t0 < kWaitLimitNs) {
    }
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTfTmemCols);
  }
}

}  // namespace

bool attn_tf32_supported(const tt_attn_args_t* a) {
  if (a->dtype != TT_F32 || (a->head_dim != 64 && a->head_dim != 128)) return false;
  // 16-byte aligned rows for the vector stores of the output
  return (reinterpret_cast<uintptr_t>(a->out) & 15u) == 0;
}

AttnPlan attn_tf32_plan(const tt_attn_args_t* /*a*/, int /*num_sms*/) {
  AttnPlan pl{};
  pl.total = kHeaderBytes;
  return pl;
}

int attn_tf32_launch(const tt_attn_args_t* a, const AttnPlan& /*plan*/, void* ws, cudaStream_t stream) {
  Tf32Params p{};
  p.q = static_cast<const float*>(a->q);
  p.k_blk = static_cast<const float*>(a->k_blk);
  p.v_blk = static_cast<const float*>(a->v_blk);
  p.k_ctx = static_cast<const float*>(a->k_ctx);
  p.v_ctx = static_cast<const float*>(a->v_ctx);
  p.ctx_lens = a->ctx_lens;
  p.page_table = a->page_table;
  p.B = a->batch;
  p.S = a->block_size;
  p.Hq = a->num_q_heads;
  p.Hkv = a->num_kv_heads;
  p.G = a->num_q_heads / a->num_kv_heads;
  p.page_size = a->page_size;
  p.max_pages = a->max_pages_per_seq;
  p.num_pages = a->num_pages;
  p.ctx_stride = a->ctx_stride;
  p.scale_log2 = a->softmax_scale * 1.4426950408889634f;
  p.out = static_cast<float*>(a->out);
  p.lse = a->lse;
  p.hdr = static_cast<WsHeader*>(ws);
  p.skip_if = a->skip_if;
  const int M = p.G * p.S;
  const dim3 grid((M + kTfRows - 1) / kTfRows, p.Hkv, p.B);
  static unsigned long long attr_done = 0;   // bit per device ordinal (< 64), set once per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TT_ERR_CUDA;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(__atomic_load_n(&attr_done, __ATOMIC_ACQUIRE) & bit)) {
    if (cudaFuncSetAttribute(attn_tf32_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)TfLayout<64>::kBytes) != cudaSuccess ||
        cudaFuncSetAttribute(attn_tf32_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)TfLayout<128>::kBytes) != cudaSuccess)
      return TT_ERR_CUDA;
    __atomic_fetch_or(&attr_done, bit, __ATOMIC_ACQ_REL);
  }
  cudaError_t e;
  if (a->head_dim == 64)
    e = launch_pdl(attn_tf32_kernel<64>, grid, dim3(kTfThreads), TfLayout<64>::kBytes, stream, p);
  else
    e = launch_pdl(attn_tf32_kernel<128>, grid, dim3(kTfThreads), TfLayout<128>::kBytes, stream, p);
  return e == cudaSuccess ? TT_OK : TT_ERR_CUDA;
}

}  // namespace tt
