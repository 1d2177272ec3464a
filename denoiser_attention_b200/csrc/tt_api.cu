// C ABI entry points: host-side argument validation, workspace sizing and dispatch to the
// sm_100a kernels. Nothing here allocates device memory or keeps mutable global state.
#include <climits>
#include <cstdio>
#include <cstring>

#include "tt_common.cuh"
#include "tt_internal.h"

namespace tt {

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The kernels index rows (batch * block_size) in 32 bits and cut the logits (rows * vocab
// elements) into CTA ranges with 64-bit products of a CTA index and the element count; these
// bounds keep both exact.
static bool rows_fit(int32_t batch, int32_t block_size) {
  return (long long)batch * (long long)block_size <= (long long)INT32_MAX;
}
static bool logits_fit(int32_t batch, int32_t block_size, int32_t vocab) {
  return (long long)batch * (long long)block_size * (long long)vocab < (1LL << 40);
}

// Predict-and-noise arguments: either an explicit keep_masked >= 0 (noise_steps == 0), or a step
// r in 1..T of the linear schedule (noise_steps = T > 0).
static bool noise_schedule_valid(int32_t keep_masked, int32_t noise_steps, int32_t noise_step) {
  if (noise_steps < 0) return false;
  if (noise_steps == 0) return keep_masked >= 0;
  return noise_step >= 1 && noise_step <= noise_steps;
}

static int validate_attn(const tt_attn_args_t* a) {
  if (!a) return TT_ERR_INVALID_ARGUMENT;
  if (a->batch < 1 || a->block_size < 1 || a->num_q_heads < 1 || a->num_kv_heads < 1 || a->head_dim < 1)
    return TT_ERR_INVALID_ARGUMENT;
  if (a->num_q_heads % a->num_kv_heads != 0) return TT_ERR_INVALID_ARGUMENT;
  if (a->dtype != TT_F32 && a->dtype != TT_BF16) return TT_ERR_INVALID_ARGUMENT;
  if (!rows_fit(a->batch, a->block_size) || !rows_fit(a->batch, a->num_kv_heads)) return TT_ERR_UNSUPPORTED;
  if (!a->q || !a->k_blk || !a->v_blk || !a->k_ctx || !a->v_ctx || !a->ctx_lens || !a->out)
    return TT_ERR_INVALID_ARGUMENT;
  if (!(a->softmax_scale > 0.f) || !(a->softmax_scale < 3.0e38f)) return TT_ERR_INVALID_ARGUMENT;
  if (a->page_table) {
    if (a->page_size < 1 || a->max_pages_per_seq < 1 || a->num_pages < 1) return TT_ERR_INVALID_ARGUMENT;
  } else {
    if (a->ctx_stride < 0) return TT_ERR_INVALID_ARGUMENT;
  }
  if (a->block_size > 64) return TT_ERR_UNSUPPORTED;
  if (a->dtype == TT_BF16 && !attn_tc_supported(a)) return TT_ERR_UNSUPPORTED;
  if (a->dtype == TT_F32 && !attn_tf32_supported(a)) return TT_ERR_UNSUPPORTED;
  return TT_OK;
}

static int validate_unmask(const tt_unmask_args_t* a) {
  if (!a) return TT_ERR_INVALID_ARGUMENT;
  if (a->batch < 1 || a->block_size < 1 || a->vocab < 1) return TT_ERR_INVALID_ARGUMENT;
  if (a->dtype != TT_F32 && a->dtype != TT_BF16) return TT_ERR_INVALID_ARGUMENT;
  if (!rows_fit(a->batch, a->block_size) || !logits_fit(a->batch, a->block_size, a->vocab))
    return TT_ERR_UNSUPPORTED;
  if (!a->logits || !a->tokens || !a->is_masked || !a->n_committed || !a->n_masked) return TT_ERR_INVALID_ARGUMENT;
  if (!(a->inv_temperature > 0.f)) return TT_ERR_INVALID_ARGUMENT;
  if (a->remaining_steps < 0) return TT_ERR_INVALID_ARGUMENT;
  if (a->exclude_mask_token && (a->mask_token_id < 0 || a->mask_token_id >= a->vocab)) return TT_ERR_INVALID_ARGUMENT;
  if (a->block_size > 1024) return TT_ERR_UNSUPPORTED;
  const int W = (a->dtype == TT_BF16) ? 8 : 4;
  if (a->vocab % W != 0 || !aligned16(a->logits)) return TT_ERR_UNSUPPORTED;
  if (a->sampler != TT_SAMPLER_CONFIDENCE && a->sampler != TT_SAMPLER_PREDICT_NOISE) return TT_ERR_INVALID_ARGUMENT;
  if (a->sampler == TT_SAMPLER_PREDICT_NOISE && !noise_schedule_valid(a->keep_masked, a->noise_steps, a->noise_step))
    return TT_ERR_INVALID_ARGUMENT;
  return TT_OK;
}

static int validate_adaln(const tt_adaln_args_t* a) {
  if (!a) return TT_ERR_INVALID_ARGUMENT;
  if (a->batch < 1 || a->hidden < 1) return TT_ERR_INVALID_ARGUMENT;
  if (a->dtype != TT_F32 && a->dtype != TT_BF16) return TT_ERR_INVALID_ARGUMENT;
  switch (a->op) {
    case TT_ADALN_COND:
      if (!a->tau || !a->w1 || !a->b1 || !a->w2 || !a->b2 || !a->w3 || !a->b3 || !a->layer_emb || !a->mod)
        return TT_ERR_INVALID_ARGUMENT;
      if (a->freq_dim < 2 || (a->freq_dim & 1) || a->mlp_width < 1) return TT_ERR_INVALID_ARGUMENT;
      if (a->freq_dim > 1024 || a->mlp_width > 1024) return TT_ERR_UNSUPPORTED;
      if ((a->freq_dim & 3) || (a->mlp_width & 3)) return TT_ERR_UNSUPPORTED;
      if (!aligned16(a->w1) || !aligned16(a->w2) || !aligned16(a->w3)) return TT_ERR_UNSUPPORTED;
      return TT_OK;
    case TT_ADALN_NORM_MODULATE:
    case TT_ADALN_GATED_RESIDUAL:
    case TT_ADALN_NORM_MODULATE_RESIDUAL: {
      const bool norm = (a->op != TT_ADALN_GATED_RESIDUAL), resid = (a->op != TT_ADALN_NORM_MODULATE);
      if (a->block_size < 1) return TT_ERR_INVALID_ARGUMENT;
      if (!a->h || !a->mod || !a->out) return TT_ERR_INVALID_ARGUMENT;
      if (norm && !a->norm_w) return TT_ERR_INVALID_ARGUMENT;
      if (resid && !a->f) return TT_ERR_INVALID_ARGUMENT;
      if (norm && !(a->eps >= 0.f)) return TT_ERR_INVALID_ARGUMENT;
      if (a->op == TT_ADALN_NORM_MODULATE_RESIDUAL && (!a->out2 || a->out2 == a->out || a->out == a->f))
        return TT_ERR_INVALID_ARGUMENT;
      const int W = (a->dtype == TT_BF16) ? 8 : 4;
      if (a->hidden % W != 0) return TT_ERR_UNSUPPORTED;
      if (!aligned16(a->h) || !aligned16(a->out) || (a->f && !aligned16(a->f))) return TT_ERR_UNSUPPORTED;
      if (a->op == TT_ADALN_NORM_MODULATE_RESIDUAL && !aligned16(a->out2)) return TT_ERR_UNSUPPORTED;
      // mod and norm_w are read as float4
      if (!aligned16(a->mod) || (a->norm_w && !aligned16(a->norm_w))) return TT_ERR_UNSUPPORTED;
      return TT_OK;
    }
    default:
      return TT_ERR_INVALID_ARGUMENT;
  }
}

static int validate_lmhead(const tt_lmhead_unmask_args_t* a) {
  if (!a) return TT_ERR_INVALID_ARGUMENT;
  if (a->batch < 1 || a->block_size < 1 || a->hidden < 1 || a->vocab < 1) return TT_ERR_INVALID_ARGUMENT;
  if (!rows_fit(a->batch, a->block_size)) return TT_ERR_UNSUPPORTED;
  if (!a->x || !a->w || !a->tokens || !a->is_masked || !a->n_committed || !a->n_masked) return TT_ERR_INVALID_ARGUMENT;
  if (!(a->inv_temperature > 0.f)) return TT_ERR_INVALID_ARGUMENT;
  if (a->sampler != TT_SAMPLER_CONFIDENCE && a->sampler != TT_SAMPLER_PREDICT_NOISE) return TT_ERR_INVALID_ARGUMENT;
  if (a->sampler == TT_SAMPLER_PREDICT_NOISE && !noise_schedule_valid(a->keep_masked, a->noise_steps, a->noise_step))
    return TT_ERR_INVALID_ARGUMENT;
  if (a->dtype != TT_BF16) return TT_ERR_UNSUPPORTED;
  if (a->hidden % 64 != 0 || a->vocab % 128 != 0 || a->block_size > 1024) return TT_ERR_UNSUPPORTED;
  if (!aligned16(a->x) || !aligned16(a->w)) return TT_ERR_UNSUPPORTED;
  return TT_OK;
}

static int validate_kv_append(const tt_kv_append_args_t* a) {
  if (!a) return TT_ERR_INVALID_ARGUMENT;
  if (a->batch < 1 || a->block_size < 1 || a->num_kv_heads < 1 || a->head_dim < 1) return TT_ERR_INVALID_ARGUMENT;
  if (a->dtype != TT_F32 && a->dtype != TT_BF16) return TT_ERR_INVALID_ARGUMENT;
  if (!a->k_new || !a->v_new || !a->k_ctx || !a->v_ctx || !a->page_table || !a->ctx_lens || !a->free_pages ||
      !a->free_count)
    return TT_ERR_INVALID_ARGUMENT;
  if (a->page_size < 1 || a->max_pages_per_seq < 1 || a->num_pages < 1) return TT_ERR_INVALID_ARGUMENT;
  const int elt = (a->dtype == TT_BF16) ? 2 : 4;
  if ((a->head_dim * elt) % 16 != 0) return TT_ERR_UNSUPPORTED;
  if (!aligned16(a->k_new) || !aligned16(a->v_new) || !aligned16(a->k_ctx) || !aligned16(a->v_ctx))
    return TT_ERR_UNSUPPORTED;
  return TT_OK;
}

// One thread waits on a barrier that nothing arrives on, with the kernels' bounded wait and the
// given limit; it gives up, records the timeout in the workspace's error word and returns.
__global__ void wait_probe_kernel(WsHeader* hdr, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
    if (!mbar_wait_bounded_for(&bar, 0, &abort_flag, limit_ns))
      report_error(hdr, TT_ERR_DEVICE_TIMEOUT, TT_DETAIL_WAIT_PROBE);
  }
}

}  // namespace tt

using namespace tt;

extern "C" {

const char* tt_status_string(int status) {
  switch (status) {
    case TT_OK: return "TT_OK";
    case TT_ERR_INVALID_ARGUMENT: return "TT_ERR_INVALID_ARGUMENT";
    case TT_ERR_UNSUPPORTED: return "TT_ERR_UNSUPPORTED";
    case TT_ERR_WORKSPACE_TOO_SMALL: return "TT_ERR_WORKSPACE_TOO_SMALL";
    case TT_ERR_CUDA: return "TT_ERR_CUDA";
    case TT_ERR_DEVICE: return "TT_ERR_DEVICE";
    case TT_ERR_DEVICE_TIMEOUT: return "TT_ERR_DEVICE_TIMEOUT";
    default: return "TT_ERR_UNKNOWN";
  }
}

int tt_version(void) { return 100; }

size_t tt_denoise_attn_workspace_bytes(const tt_attn_args_t* a) {
  if (validate_attn(a) != TT_OK) return 0;
  const int sms = device_sm_count();
  return a->dtype == TT_BF16 ? attn_tc_plan(a, sms).total : attn_tf32_plan(a, sms).total;
}

int tt_denoise_attn(const tt_attn_args_t* a, void* ws, size_t ws_bytes, tt_stream_t stream) {
  const int st = validate_attn(a);
  if (st != TT_OK) return st;
  if (!ws) return TT_ERR_INVALID_ARGUMENT;
  const int sms = device_sm_count();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (a->dtype == TT_BF16) {
    const AttnPlan pl = attn_tc_plan(a, sms);
    if (ws_bytes < pl.total) return TT_ERR_WORKSPACE_TOO_SMALL;
    return attn_tc_launch(a, pl, ws, s);
  }
  const AttnPlan pl = attn_tf32_plan(a, sms);
  if (ws_bytes < pl.total) return TT_ERR_WORKSPACE_TOO_SMALL;
  return attn_tf32_launch(a, pl, ws, s);
}

size_t tt_adaln_workspace_bytes(const tt_adaln_args_t* a) {
  if (validate_adaln(a) != TT_OK) return 0;
  return adaln_workspace_bytes(a);
}

int tt_adaln_modulate(const tt_adaln_args_t* a, void* ws, size_t ws_bytes, tt_stream_t stream) {
  const int st = validate_adaln(a);
  if (st != TT_OK) return st;
  if (!ws) return TT_ERR_INVALID_ARGUMENT;
  if (ws_bytes < adaln_workspace_bytes(a)) return TT_ERR_WORKSPACE_TOO_SMALL;
  return adaln_launch(a, ws, reinterpret_cast<cudaStream_t>(stream));
}

size_t tt_unmask_workspace_bytes(const tt_unmask_args_t* a) {
  if (validate_unmask(a) != TT_OK) return 0;
  return unmask_plan(a, device_sm_count()).layout.total;
}

int tt_unmask_step(const tt_unmask_args_t* a, void* ws, size_t ws_bytes, tt_stream_t stream) {
  const int st = validate_unmask(a);
  if (st != TT_OK) return st;
  if (!ws) return TT_ERR_INVALID_ARGUMENT;
  const UnmaskPlan pl = unmask_plan(a, device_sm_count());
  if (ws_bytes < pl.layout.total) return TT_ERR_WORKSPACE_TOO_SMALL;
  return unmask_launch(a, pl, ws, reinterpret_cast<cudaStream_t>(stream));
}

int tt_unmask_step_noalloc(const tt_unmask_args_t* a, tt_stream_t stream) {
  const int st = validate_unmask(a);
  if (st != TT_OK) return st;
  return unmask_launch_static(a, reinterpret_cast<cudaStream_t>(stream));
}

int tt_block_tau(const uint8_t* is_masked, int32_t batch, int32_t block_size, float* tau, const int32_t* skip_if,
                 tt_stream_t stream) {
  if (!is_masked || !tau || batch < 1 || block_size < 1) return TT_ERR_INVALID_ARGUMENT;
  return block_tau_launch(is_masked, batch, block_size, tau, skip_if, reinterpret_cast<cudaStream_t>(stream));
}

size_t tt_lmhead_unmask_workspace_bytes(const tt_lmhead_unmask_args_t* a) {
  return validate_lmhead(a) == TT_OK ? lmhead_workspace_bytes(a, device_sm_count()) : 0;
}

int tt_lmhead_unmask_step(const tt_lmhead_unmask_args_t* a, void* ws, size_t ws_bytes, tt_stream_t stream) {
  const int st = validate_lmhead(a);
  if (st != TT_OK) return st;
  if (!ws) return TT_ERR_INVALID_ARGUMENT;
  if (ws_bytes < lmhead_workspace_bytes(a, device_sm_count())) return TT_ERR_WORKSPACE_TOO_SMALL;
  return lmhead_unmask_launch(a, ws, reinterpret_cast<cudaStream_t>(stream));
}

size_t tt_kv_append_workspace_bytes(const tt_kv_append_args_t* a) {
  return validate_kv_append(a) == TT_OK ? kHeaderBytes : 0;
}

int tt_kv_append(const tt_kv_append_args_t* a, void* ws, size_t ws_bytes, tt_stream_t stream) {
  const int st = validate_kv_append(a);
  if (st != TT_OK) return st;
  if (!ws) return TT_ERR_INVALID_ARGUMENT;
  if (ws_bytes < kHeaderBytes) return TT_ERR_WORKSPACE_TOO_SMALL;
  return kv_append_launch(a, ws, reinterpret_cast<cudaStream_t>(stream));
}

int32_t tt_linear_schedule_keep(int32_t block_size, int32_t steps, int32_t step) {
  if (block_size < 1 || steps < 1 || step < 1 || step > steps) return -1;
  return linear_schedule_keep(block_size, steps, step);
}

int tt_probe_bounded_wait(void* ws, uint32_t limit_us, tt_stream_t stream) {
  if (!ws || limit_us < 1 || limit_us > 1000000u) return TT_ERR_INVALID_ARGUMENT;
  wait_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(static_cast<WsHeader*>(ws),
                                                                           (uint64_t)limit_us * 1000ull);
  return cudaGetLastError() == cudaSuccess ? TT_OK : TT_ERR_CUDA;
}

int tt_get_device_error(void* ws, tt_stream_t stream, uint32_t* detail) {
  if (!ws) return TT_ERR_INVALID_ARGUMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t host[2] = {0, 0};
  if (cudaMemcpyAsync(host, ws, sizeof(host), cudaMemcpyDeviceToHost, s) != cudaSuccess) return TT_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return TT_ERR_CUDA;
  if (host[0] != 0) {
    if (cudaMemsetAsync(ws, 0, sizeof(host), s) != cudaSuccess) return TT_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return TT_ERR_CUDA;
  }
  if (detail) *detail = host[1];
  return (int)host[0];
}

}  // extern "C"
