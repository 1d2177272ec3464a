// Host-side interfaces between the C ABI layer (tt_api.cu) and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/tt_denoise.h"

namespace tt {

// ---------------------------------------------------------------- unmask
struct UnmaskLayout {
  size_t row_cnt, seq_cnt, done, partials, conf, argmax, total;
};
struct UnmaskPlan {
  int grid;            // CTAs, each streaming an equal share of the logits
  UnmaskLayout layout;
};
UnmaskPlan unmask_plan(const tt_unmask_args_t* a, int num_sms);
int unmask_launch(const tt_unmask_args_t* a, const UnmaskPlan& plan, void* ws, cudaStream_t stream);
// Same launch with the module's static scratch (no allocation, no caller workspace).
int unmask_launch_static(const tt_unmask_args_t* a, cudaStream_t stream);
// The unmask step from hidden states through the LM head (logits never stored).
size_t lmhead_workspace_bytes(const tt_lmhead_unmask_args_t* a, int num_sms);
int lmhead_unmask_launch(const tt_lmhead_unmask_args_t* a, void* ws, cudaStream_t stream);
// Linear noise schedule of the predict-and-noise sampler: positions left masked after step r of T.
inline int32_t linear_schedule_keep(int32_t S, int32_t T, int32_t r) {
  return (int32_t)(((long long)S * (long long)(T - r)) / (long long)T);
}
// keep_masked of a predict-and-noise call: derived from the schedule when noise_steps > 0.
inline int32_t predict_noise_keep(int32_t S, int32_t keep_masked, int32_t noise_steps, int32_t noise_step) {
  return noise_steps > 0 ? linear_schedule_keep(S, noise_steps, noise_step) : keep_masked;
}
// tau[b] = masked positions of sequence b / S.
int block_tau_launch(const uint8_t* is_masked, int B, int S, float* tau, const int32_t* skip_if,
                     cudaStream_t stream);

// ---------------------------------------------------------------- block commit (paged KV append)
int kv_append_launch(const tt_kv_append_args_t* a, void* ws, cudaStream_t stream);

// ---------------------------------------------------------------- adaLN
size_t adaln_workspace_bytes(const tt_adaln_args_t* a);
int adaln_launch(const tt_adaln_args_t* a, void* ws, cudaStream_t stream);

// ---------------------------------------------------------------- attention
struct AttnPlan {
  int grid;            // persistent CTAs
  int qtiles;          // query-row tiles per (sequence, kv head)
  int team_size;       // CTAs per team (two-stream kernel: up to two query tiles of a group per CTA)
  int one_tile;        // 1: attn_tc1_kernel, one query tile per CTA (teams of qtiles CTAs)
  int s_per_tile;      // block positions per query-row tile
  int units;           // groups: batch * kv heads
  size_t off_meta;     // total tiles and working CTAs of the partition
  size_t off_crange;   // int32 [units][2]: first and last team holding each unit's partials
  size_t off_partials; // float [slots][rows][d]
  size_t off_lse;      // float [slots][rows]
  size_t slots;
  size_t total;
};
bool attn_tc_supported(const tt_attn_args_t* a);
AttnPlan attn_tc_plan(const tt_attn_args_t* a, int num_sms);
int attn_tc_launch(const tt_attn_args_t* a, const AttnPlan& plan, void* ws, cudaStream_t stream);

bool attn_tf32_supported(const tt_attn_args_t* a);
AttnPlan attn_tf32_plan(const tt_attn_args_t* a, int num_sms);
int attn_tf32_launch(const tt_attn_args_t* a, const AttnPlan& plan, void* ws, cudaStream_t stream);

int device_sm_count();

}  // namespace tt
