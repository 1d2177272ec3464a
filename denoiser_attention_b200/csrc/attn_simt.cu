// Eq. (1) of "Nemotron-TwoTower: Diffusion Language Modeling with Pretrained AR Context" (§2.1,
// "Bidirectional attention") for fp32 tensors, on the CUDA cores.
//
// fp32 inputs carry a 1e-5 accuracy bar that tensor-core tf32 cannot meet, and the fp32
// workloads are small, so this path uses plain fp32 FMA. One CTA owns 64 query rows of one
// (sequence, kv head): rows m = s * G + g (block position s, query head kvh * G + g). Keys are
// streamed in tiles of 32 through shared memory (context tokens through the page table, then
// the block's own S tokens); each warp keeps an online softmax (m, l, o) for 8 rows.
#include <cmath>

#include "tt_common.cuh"
#include "tt_internal.h"

namespace tt {

constexpr int kSimtThreads = 256;
constexpr int kSimtRows = 64;     // query rows per CTA
constexpr int kSimtKeys = 32;     // keys per tile

struct SimtParams {
  const float* q;
  const float* k_blk;
  const float* v_blk;
  const float* k_ctx;
  const float* v_ctx;
  const int32_t* ctx_lens;
  const int32_t* page_table;
  int32_t B, S, Hq, Hkv, G, d;
  int32_t page_size, max_pages, num_pages, ctx_stride;
  float scale;
  float* out;
  float* lse;
  WsHeader* hdr;
};

template <int D>
__global__ void __launch_bounds__(kSimtThreads) attn_simt_kernel(const SimtParams p) {
  constexpr int DP = D + 1;            // padded row (conflict-free column reads)
  constexpr int PER_LANE = D / 32;
  extern __shared__ float smem[];
  float* s_q = smem;                                   // [64][D]
  float* s_k = s_q + kSimtRows * D;                    // [32][DP]
  float* s_v = s_k + kSimtKeys * DP;                   // [32][DP]
  __shared__ int s_row[kSimtKeys];                     // source row of each tile key (-1: none)
  pdl_trigger();
  pdl_wait();

  const int b = blockIdx.z, kvh = blockIdx.y;
  const int row0 = blockIdx.x * kSimtRows;
  const int M = p.G * p.S;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  int L = p.ctx_lens[b];
  if (L < 0) {
    if (tid == 0) report_error(p.hdr, TT_ERR_DEVICE, kDetailNegativeLen);
    L = 0;
  }
  const int cap = p.page_table ? p.max_pages * p.page_size : p.ctx_stride;
  if (L > cap) {
    if (tid == 0) report_error(p.hdr, TT_ERR_DEVICE, kDetailCtxTooLong);
    L = cap;
  }

  // query rows of this CTA
  for (int i = tid; i < kSimtRows * D; i += blockDim.x) {
    const int r = i / D, c = i - r * D;
    const int m = row0 + r;
    float v = 0.f;
    if (m < M) {
      const int s = m / p.G, g = m - s * p.G;
      v = p.q[(((size_t)b * p.S + s) * p.Hq + kvh * p.G + g) * D + c];
    }
    s_q[i] = v;
  }

  float mrun[8], lrun[8], o[8][PER_LANE];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    mrun[r] = -INFINITY;
    lrun[r] = 0.f;
#pragma unroll
    for (int k = 0; k < PER_LANE; ++k) o[r][k] = 0.f;
  }

  const int total = L + p.S;
  for (int t0 = 0; t0 < total; t0 += kSimtKeys) {
    __syncthreads();
    if (tid < kSimtKeys) {
      const int t = t0 + tid;
      int src = -1;   // >= 0: context row index into k_ctx rows; <= -2: block row -(src+2)
      if (t < L) {
        if (p.page_table) {
          const int pg = p.page_table[(size_t)b * p.max_pages + t / p.page_size];
          if (pg < 0 || pg >= p.num_pages) {
            report_error(p.hdr, TT_ERR_DEVICE, kDetailBadPage);
          } else {
            src = pg * p.page_size + t % p.page_size;
          }
        } else {
          src = b * p.ctx_stride + t;
        }
      } else if (t < total) {
        src = -2 - (b * p.S + (t - L));
      }
      s_row[tid] = src;
    }
    __syncthreads();
    for (int i = tid; i < kSimtKeys * D; i += blockDim.x) {
      const int j = i / D, c = i - j * D;
      const int src = s_row[j];
      float kv = 0.f, vv = 0.f;
      if (src >= 0) {
        const size_t off = ((size_t)src * p.Hkv + kvh) * D + c;
        kv = p.k_ctx[off];
        vv = p.v_ctx[off];
      } else if (src <= -2) {
        const size_t off = ((size_t)(-2 - src) * p.Hkv + kvh) * D + c;
        kv = p.k_blk[off];
        vv = p.v_blk[off];
      }
      s_k[j * DP + c] = kv;
      s_v[j * DP + c] = vv;
    }
    __syncthreads();
    const bool key_ok = (s_row[lane] != -1) && (t0 + lane < total);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int lr = warp * 8 + r;
      const float* qr = s_q + lr * D;
      float dot = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) dot = fmaf(qr[c], s_k[lane * DP + c], dot);
      const float x = key_ok ? dot * p.scale : -INFINITY;
      float tmax = x;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
      const float mnew = fmaxf(mrun[r], tmax);
      const float corr = (mrun[r] == -INFINITY) ? 0.f : expf(mrun[r] - mnew);
      const float pj = key_ok ? expf(x - mnew) : 0.f;
      float psum = pj;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
      lrun[r] = lrun[r] * corr + psum;
      mrun[r] = mnew;
#pragma unroll
      for (int k = 0; k < PER_LANE; ++k) o[r][k] *= corr;
      for (int j = 0; j < kSimtKeys; ++j) {
        const float pjj = __shfl_sync(0xffffffffu, pj, j);
#pragma unroll
        for (int k = 0; k < PER_LANE; ++k) o[r][k] = fmaf(pjj, s_v[j * DP + lane + 32 * k], o[r][k]);
      }
    }
  }

#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int m = row0 + warp * 8 + r;
    if (m >= M) continue;
    const int s = m / p.G, g = m - s * p.G;
    const int h = kvh * p.G + g;
    const float inv = 1.0f / lrun[r];
    float* dst = p.out + (((size_t)b * p.S + s) * p.Hq + h) * D;
#pragma unroll
    for (int k = 0; k < PER_LANE; ++k) dst[lane + 32 * k] = o[r][k] * inv;
    if (p.lse && lane == 0) p.lse[((size_t)b * p.Hq + h) * p.S + s] = mrun[r] + logf(lrun[r]);
  }
}

bool attn_simt_supported(const tt_attn_args_t* a) {
  return a->dtype == TT_F32 && (a->head_dim == 64 || a->head_dim == 128);
}

AttnPlan attn_simt_plan(const tt_attn_args_t* a, int /*num_sms*/) {
  AttnPlan pl{};
  pl.total = kHeaderBytes;
  return pl;
}

int attn_simt_launch(const tt_attn_args_t* a, const AttnPlan& /*plan*/, void* ws, cudaStream_t stream) {
  SimtParams p{};
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
  p.d = a->head_dim;
  p.page_size = a->page_size;
  p.max_pages = a->max_pages_per_seq;
  p.num_pages = a->num_pages;
  p.ctx_stride = a->ctx_stride;
  p.scale = a->softmax_scale;
  p.out = static_cast<float*>(a->out);
  p.lse = a->lse;
  p.hdr = static_cast<WsHeader*>(ws);
  const int M = p.G * p.S;
  dim3 grid((M + kSimtRows - 1) / kSimtRows, p.Hkv, p.B);
  static unsigned long long attr_done = 0;   // bit per device ordinal (< 64), set once per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TT_ERR_CUDA;
  const unsigned long long bit = 1ull << (dev & 63);
  const size_t smem64 = sizeof(float) * (kSimtRows * 64 + 2 * kSimtKeys * 65);
  const size_t smem128 = sizeof(float) * (kSimtRows * 128 + 2 * kSimtKeys * 129);
  if (!(__atomic_load_n(&attr_done, __ATOMIC_ACQUIRE) & bit)) {
    if (cudaFuncSetAttribute(attn_simt_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem64) !=
            cudaSuccess ||
        cudaFuncSetAttribute(attn_simt_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem128) !=
            cudaSuccess)
      return TT_ERR_CUDA;
    __atomic_fetch_or(&attr_done, bit, __ATOMIC_ACQ_REL);
  }
  if (p.d == 64)
    launch_pdl(attn_simt_kernel<64>, grid, dim3(kSimtThreads), smem64, stream, p);
  else
    launch_pdl(attn_simt_kernel<128>, grid, dim3(kSimtThreads), smem128, stream, p);
  return cudaGetLastError() == cudaSuccess ? TT_OK : TT_ERR_CUDA;
}

}  // namespace tt
