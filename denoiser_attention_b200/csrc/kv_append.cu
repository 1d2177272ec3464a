// Block commit into the paged context cache: the context update of Algorithm 1 in "Nemotron-TwoTower:
// Diffusion Language Modeling with Pretrained AR Context" (§2.2 "Sampling"): once block b is committed, the
// context tower's KV of its S tokens joins the prefix cache that the next block's denoiser
// attention reads. The context tower itself (which produces that KV) is not part of this path;
// this kernel appends the rows it produced and grows the page tables.
//
// One CTA per sequence. Thread 0 takes the pages the block newly needs from a device-side stack of
// free page ids (a compare-and-swap on the stack count) and enters them in the page table; then the
// CTA copies the S x Hkv rows of K and V into their page slots with 16-byte vector copies and
// advances ctx_lens[b] by S. A sequence whose pages cannot be provided (stack exhausted, page
// table full) is left unchanged and the workspace error word is set.
#include "tt_common.cuh"
#include "tt_internal.h"

namespace tt {

namespace {

constexpr int kAppendThreads = 256;
constexpr int kMaxClaimRounds = 1 << 20;

struct AppendParams {
  const uint4* k_new;
  const uint4* v_new;
  uint4* k_ctx;
  uint4* v_ctx;
  int32_t* page_table;
  int32_t* ctx_lens;
  const int32_t* free_pages;
  int32_t* free_count;
  int32_t S, Hkv, vec_per_row;   // 16-byte vectors per (token, head) row = head_dim * elt / 16
  int32_t page_size, max_pages, num_pages;
  WsHeader* hdr;
};

__global__ void __launch_bounds__(kAppendThreads) kv_append_kernel(const AppendParams p) {
  __shared__ int s_ok;
  __shared__ int s_len;
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  if (tid == 0) {
    int L = p.ctx_lens[b];
    int ok = 1;
    if (L < 0) {
      report_error(p.hdr, TT_ERR_DEVICE, kDetailNegativeLen);
      ok = 0;
    }
    const long long have = ((long long)L + p.page_size - 1) / p.page_size;          // pages holding tokens
    const long long need = ((long long)L + p.S + p.page_size - 1) / p.page_size;    // after the append
    if (ok && need > p.max_pages) {
      report_error(p.hdr, TT_ERR_DEVICE, kDetailPageTableFull);
      ok = 0;
    }
    if (ok && need > have) {
      // Claim the top n entries of the free stack with a compare-and-swap that only ever moves
      // the count from `top` to `top - n` when top >= n: a claim that cannot be served never
      // changes the count, so concurrent failures cannot expose pages another sequence holds.
      // The entries a claim would take are checked before the swap (the stack array is not
      // written during the launch), so a bad page id leaves this sequence and the stack as they
      // were. Every failed swap means another sequence's swap succeeded, so the loop ends within
      // `batch` rounds; the bound below only guards against a count written concurrently by
      // something outside this launch.
      const int n = (int)(need - have);
      int top = *reinterpret_cast<volatile int*>(p.free_count);
      ok = 0;
      bool settled = false;   // claimed, or failed with an error reported
      for (int attempt = 0; attempt < kMaxClaimRounds && !settled; ++attempt) {
        if (top < n) {
          report_error(p.hdr, TT_ERR_DEVICE, kDetailOutOfPages);
          settled = true;
          break;
        }
        bool valid = true;
        for (int i = 0; i < n; ++i) {
          const int pg = p.free_pages[top - n + i];
          valid = valid && pg >= 0 && pg < p.num_pages;
        }
        if (!valid) {
          report_error(p.hdr, TT_ERR_DEVICE, kDetailBadPage);
          settled = true;
          break;
        }
        const int prev = atomicCAS(p.free_count, top, top - n);
        if (prev == top) {
          for (int i = 0; i < n; ++i)
            p.page_table[(size_t)b * p.max_pages + have + i] = p.free_pages[top - n + i];
          ok = 1;
          settled = true;
          break;
        }
        top = prev;
      }
      if (!settled) report_error(p.hdr, TT_ERR_DEVICE, kDetailClaimContended);
    }
    s_ok = ok;
    s_len = L;
  }
  __syncthreads();
  if (!s_ok) return;
  const int L = s_len;
  // rows (r, h) of the block, each vec_per_row 16-byte vectors
  const int per_tok = p.Hkv * p.vec_per_row;
  const int total = p.S * per_tok;
  for (int i = tid; i < total; i += kAppendThreads) {
    const int r = i / per_tok, rem = i - r * per_tok;
    const int pos = L + r;
    const int pg = p.page_table[(size_t)b * p.max_pages + pos / p.page_size];
    const size_t dst = ((size_t)pg * p.page_size + pos % p.page_size) * per_tok + rem;
    const size_t src = ((size_t)b * p.S + r) * per_tok + rem;
    p.k_ctx[dst] = p.k_new[src];
    p.v_ctx[dst] = p.v_new[src];
  }
  if (tid == 0) p.ctx_lens[b] = L + p.S;
}

}  // namespace

int kv_append_launch(const tt_kv_append_args_t* a, void* ws, cudaStream_t stream) {
  const int elt = (a->dtype == TT_BF16) ? 2 : 4;
  AppendParams p{};
  p.k_new = static_cast<const uint4*>(a->k_new);
  p.v_new = static_cast<const uint4*>(a->v_new);
  p.k_ctx = static_cast<uint4*>(a->k_ctx);
  p.v_ctx = static_cast<uint4*>(a->v_ctx);
  p.page_table = a->page_table;
  p.ctx_lens = a->ctx_lens;
  p.free_pages = a->free_pages;
  p.free_count = a->free_count;
  p.S = a->block_size;
  p.Hkv = a->num_kv_heads;
  p.vec_per_row = a->head_dim * elt / 16;
  p.page_size = a->page_size;
  p.max_pages = a->max_pages_per_seq;
  p.num_pages = a->num_pages;
  p.hdr = static_cast<WsHeader*>(ws);
  return launch_pdl(kv_append_kernel, dim3(a->batch), dim3(kAppendThreads), 0, stream, p) == cudaSuccess ? TT_OK
                                                                                                       : TT_ERR_CUDA;
}

}  // namespace tt
