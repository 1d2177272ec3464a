// Eq. (1) of "Nemotron-TwoTower: Diffusion Language Modeling with Pretrained AR Context"
// (§2.1 "Bidirectional attention") for bf16 tensors on the sm_100a tensor cores.
//
// Work decomposition. A "unit" is (sequence b, kv head, query-row tile). Its query rows are the
// G query heads of the kv head times the block positions of the tile, packed as M rows
// m = s * G + g (at most 256 = two 128-row MMA halves), so each key/value tile is read from HBM
// once per unit. Its keys are ceil(L_b/64) context tiles of 64 tokens followed by one tile holding
// the S block tokens. All units' tiles are laid end to end and cut into Pe = min(gridDim.x, tiles)
// equal ranges, one per persistent CTA (one CTA per SM), so ragged contexts are balanced to within
// a tile without any host-side knowledge of the lengths. A CTA that holds a whole unit writes its
// output directly; a unit cut between CTAs leaves one normalised partial (O_j / l_j and the
// log2-sum-exp) per CTA, and a second, wide kernel merges them (flash-decoding combine). The
// merge kernel is launched as a programmatic dependent of the attention kernel, so its launch
// overlaps the attention tail and it starts reading partials as soon as they are complete.
//
// Inside a CTA (384 threads):
//   warp 0      TMA producer: Q tile of the unit, then K/V tiles into a 4-stage ring
//               (128B-swizzled boxes of 64 tokens x 64 dims; no multicast)
//   warp 1      MMA issuer (one thread): S_h = Q_h K^T (M=128, N=64, K=128) into TMEM, then
//               O_h += P_h V (M=128, N=128, K=64) with P read from TMEM; QK^T of tile f+1 is
//               issued before PV of tile f so the tensor pipe works while the softmax runs
//   warps 4-7   softmax + epilogue for rows 0..127 (thread = TMEM lane = row)
//   warps 8-11  softmax + epilogue for rows 128..255
// TMEM (512 columns): O_0 [0,128), O_1 [128,256), S/P double buffers of 64 columns per half.
// The softmax works in the exp2 domain with the scale folded in; the running maximum used for
// the exponentials is only raised when a tile's maximum exceeds it by more than 8 (a factor 256),
// which keeps the O rescale off the common path and stays exact because numerator and
// denominator use the same stale maximum. Only a rescale waits for the previous PV product.
#include <cstdio>
#include <cuda.h>
#include <cudaTypedefs.h>

#include "tt_common.cuh"
#include "tt_internal.h"

namespace tt {

namespace {

constexpr int kD = 128;           // head dim handled by this kernel
constexpr int kTile = 64;         // keys per tile
constexpr int kStages = 4;        // K/V ring depth
constexpr int kThreads = 384;
constexpr int kRowsPerHalf = 128;
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kQBytesPerDh = 256 * 128;                   // 256 rows x 128 B
constexpr uint32_t kQBytes = 2 * kQBytesPerDh;                 // 64 KB
constexpr uint32_t kKVBoxBytes = kTile * 128;                  // 64 rows x 128 B = 8 KB
constexpr uint32_t kKBytesPerStage = 2 * kKVBoxBytes;          // 16 KB
constexpr uint32_t kStageBytes = 2 * kKBytesPerStage;          // K + V = 32 KB
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemK = kQBytes;
constexpr uint32_t kSmemV = kSmemK + kStages * kKBytesPerStage;
constexpr uint32_t kSmemBar = kSmemV + kStages * kKBytesPerStage;
constexpr uint32_t kSmemBytes = kSmemBar + 1024 + 1024;        // barriers/scratch + alignment slack

constexpr int kMergeRows = 32;    // rows per merge CTA (8 warps x 4 rows)

// Instruction descriptors (kind::f16): D fp32, A/B bf16, A K-major.
constexpr uint32_t make_idesc(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}
constexpr uint32_t kIdescQK = make_idesc(128, kTile, false);
constexpr uint32_t kIdescPV = make_idesc(128, kD, true);

// Shared-memory matrix descriptor, 128-byte swizzle.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;   // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;   // SWIZZLE_128B
  return d;
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Workspace: header | meta (total tiles, working CTAs) | unit_start[units + 1] | partials | lse
struct AttnMeta {
  long long total_tiles;
  long long p_eff;
};

struct TcParams {
  CUtensorMap tm_q, tm_kc, tm_vc, tm_kb, tm_vb;
  const int32_t* ctx_lens;
  const int32_t* page_table;
  int32_t B, S, Hq, Hkv, G;
  int32_t qtiles, s_per_tile, units;
  int32_t page_size, max_pages, num_pages, ctx_stride, paged;
  float scale_log2;   // softmax_scale * log2(e)
  __nv_bfloat16* out;
  float* lse;
  uint8_t* ws;
  size_t off_meta, off_ustart, off_partials, off_lse;
};

struct Smem {
  uint64_t q_full, q_empty;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2][2], p_full[2][2], pv_done[2][2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  long long range_begin, range_end, total_tiles, p_eff;
  int u0;
  long long u0_start;
};

struct UnitInfo {
  int b, kvh, qt, L, nctx, ntiles;
};

__device__ __forceinline__ int clamp_len(const int32_t* ctx_lens, int paged, int max_pages, int page_size,
                                         int ctx_stride, int b, bool report, WsHeader* hdr) {
  int L = ctx_lens[b];
  if (L < 0) {
    if (report) report_error(hdr, TT_ERR_DEVICE, kDetailNegativeLen);
    L = 0;
  }
  const int cap = paged ? max_pages * page_size : ctx_stride;
  if (L > cap) {
    if (report) report_error(hdr, TT_ERR_DEVICE, kDetailCtxTooLong);
    L = cap;
  }
  return L;
}

__device__ __forceinline__ UnitInfo unit_info(const TcParams& p, int u, bool report, WsHeader* hdr) {
  UnitInfo ui;
  ui.qt = u % p.qtiles;
  const int bk = u / p.qtiles;
  ui.kvh = bk % p.Hkv;
  ui.b = bk / p.Hkv;
  ui.L = clamp_len(p.ctx_lens, p.paged, p.max_pages, p.page_size, p.ctx_stride, ui.b, report, hdr);
  ui.nctx = (ui.L + kTile - 1) / kTile;
  ui.ntiles = ui.nctx + 1;
  return ui;
}

// Walks the units overlapping this CTA's tile range, one segment (a maximal run of tiles of one
// unit) at a time. Every role runs its own copy; all copies see the same sequence.
struct SegWalk {
  int u;
  long long ustart;
  long long g, gend;
  UnitInfo ui;
  __device__ void init(const TcParams& p, const Smem& sm, WsHeader* hdr) {
    u = sm.u0;
    ustart = sm.u0_start;
    g = sm.range_begin;
    gend = sm.range_end;
    ui = unit_info(p, u, false, hdr);
  }
  __device__ bool done() const { return g >= gend; }
  // tiles [kb, ke) of unit ui in the current segment
  __device__ void segment(int& kb, int& ke) const {
    kb = (int)(g - ustart);
    const long long uend = ustart + ui.ntiles;
    ke = (int)((uend < gend ? uend : gend) - ustart);
  }
  __device__ void advance(const TcParams& p, WsHeader* hdr) {
    int kb, ke;
    segment(kb, ke);
    g = ustart + ke;
    if (ke == ui.ntiles && g < gend) {
      ustart += ui.ntiles;
      ++u;
      ui = unit_info(p, u, false, hdr);
    }
  }
};

// CTA index owning global tile t when T tiles are cut into P <= T ranges [c*T/P, (c+1)*T/P).
__device__ __forceinline__ long long owner_cta(long long t, long long T, long long P) {
  return ((t + 1) * P - 1) / T;
}

__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem& sm = *reinterpret_cast<Smem*>(smem + kSmemBar);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(p.ws);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long P = gridDim.x, cta = blockIdx.x;

  // ---- 0. prologue that touches no input: barriers, TMEM, tensor-map prefetch. With a
  // programmatic launch it overlaps the previous kernel; inputs are read after pdl_wait().
  if (warp == 0 && lane == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.kv_full[i], 1);
      mbar_init(&sm.kv_empty[i], 1);
    }
    for (int h = 0; h < 2; ++h) {
      for (int bf = 0; bf < 2; ++bf) {
        mbar_init(&sm.s_full[h][bf], 1);
        mbar_init(&sm.p_full[h][bf], kRowsPerHalf);
        mbar_init(&sm.pv_done[h][bf], 1);
      }
    }
    mbar_init(&sm.drain, 1);
    fence_barrier_init();
    prefetch_tmap(&p.tm_q);
    prefetch_tmap(&p.tm_kc);
    prefetch_tmap(&p.tm_vc);
    prefetch_tmap(&p.tm_kb);
    prefetch_tmap(&p.tm_vb);
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  pdl_trigger();
  pdl_wait();

  // ---- 1. this CTA's tile range and the unit where it starts (warp 0); CTA 0 also records the
  // partition for the merge kernel
  if (warp == 0) {
    long long T = 0;
    for (int base = 0; base < p.units; base += 32) {
      const int u = base + lane;
      int n = 0;
      if (u < p.units) n = unit_info(p, u, blockIdx.x == 0, hdr).ntiles;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
      T += n;
    }
    // with fewer tiles than CTAs only the first T CTAs work (one tile each), so every working
    // CTA owns a non-empty range and the CTAs of a unit are consecutive
    const long long Pe = T < P ? T : P;
    const long long rb = cta < Pe ? cta * T / Pe : T, re = cta < Pe ? (cta + 1) * T / Pe : T;
    long long acc = 0;
    int u0 = -1;
    long long u0s = 0;
    int32_t* ustart_out = reinterpret_cast<int32_t*>(p.ws + p.off_ustart);
    const bool record = (blockIdx.x == 0);
    for (int base = 0; base < p.units && (u0 < 0 || record); base += 32) {
      const int u = base + lane;
      const int n = (u < p.units) ? unit_info(p, u, false, hdr).ntiles : 0;
      int incl = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const long long lo = acc + incl - n, hi = acc + incl;
      if (record && u < p.units) ustart_out[u] = (int32_t)lo;
      const unsigned hit = __ballot_sync(0xffffffffu, u < p.units && lo <= rb && rb < hi);
      if (hit && u0 < 0) {
        const int src = __ffs(hit) - 1;
        u0 = base + src;
        u0s = __shfl_sync(0xffffffffu, lo, src);
      }
      acc += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      sm.total_tiles = T;
      sm.p_eff = Pe;
      sm.range_begin = rb;
      sm.range_end = re;
      sm.u0 = u0;
      sm.u0_start = u0s;
      sm.abort_flag = 0;
      if (record) {
        ustart_out[p.units] = (int32_t)T;
        AttnMeta* meta = reinterpret_cast<AttnMeta*>(p.ws + p.off_meta);
        meta->total_tiles = T;
        meta->p_eff = Pe;
      }
    }
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;
  const bool has_work = sm.range_begin < sm.range_end && sm.u0 >= 0;

  const int M = p.G * p.s_per_tile;               // query rows per unit (<= 256)
  const int nh = (M > kRowsPerHalf) ? 2 : 1;      // active 128-row halves

  auto fail = [&](uint32_t detail) {
    report_error(hdr, TT_ERR_DEVICE_TIMEOUT, detail);
    *abort_flag = 1;
  };

  const uint32_t sQ = smem_u32(smem + kSmemQ);
  const uint32_t sK = smem_u32(smem + kSmemK);
  const uint32_t sV = smem_u32(smem + kSmemV);

  if (!has_work) {
    // nothing to do (more CTAs than tiles)
  } else if (warp == 0) {
    // ======================= TMA producer
    if (lane == 0) {
      SegWalk w;
      w.init(p, sm, hdr);
      long long f = 0;
      int qn = 0;
      bool ok = true;
      const uint32_t q_bytes = 2u * 128u * (uint32_t)p.G * (uint32_t)p.s_per_tile;
      while (ok && !w.done()) {
        int kb, ke;
        w.segment(kb, ke);
        const UnitInfo& ui = w.ui;
        if (qn > 0 && !mbar_wait_bounded(&sm.q_empty, (qn - 1) & 1, abort_flag)) {
          fail(kDetailWaitQEmpty);
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&sm.q_full, q_bytes);
        const int qrow = ui.b * p.S + ui.qt * p.s_per_tile;
        tma_load_3d(smem + kSmemQ, &p.tm_q, &sm.q_full, 0, ui.kvh * p.G, qrow);
        tma_load_3d(smem + kSmemQ + kQBytesPerDh, &p.tm_q, &sm.q_full, 64, ui.kvh * p.G, qrow);
        ++qn;
        for (int k = kb; k < ke; ++k, ++f) {
          const int stage = (int)(f % kStages);
          const long long round = f / kStages;
          if (round > 0 && !mbar_wait_bounded(&sm.kv_empty[stage], (uint32_t)((round - 1) & 1), abort_flag)) {
            fail(kDetailWaitKvEmpty);
            ok = false;
            break;
          }
          const CUtensorMap* mk;
          const CUtensorMap* mv;
          int row;
          if (k < ui.nctx) {
            const int t0 = k * kTile;
            if (p.paged) {
              int pg = p.page_table[(size_t)ui.b * p.max_pages + t0 / p.page_size];
              if (pg < 0 || pg >= p.num_pages) {
                report_error(hdr, TT_ERR_DEVICE, kDetailBadPage);
                pg = 0;   // read a valid page instead; the result is unspecified, the error is set
              }
              row = pg * p.page_size + t0 % p.page_size;
            } else {
              row = ui.b * p.ctx_stride + t0;
            }
            mk = &p.tm_kc;
            mv = &p.tm_vc;
          } else {
            row = ui.b * p.S;
            mk = &p.tm_kb;
            mv = &p.tm_vb;
          }
          uint8_t* kdst = smem + kSmemK + stage * kKBytesPerStage;
          uint8_t* vdst = smem + kSmemV + stage * kKBytesPerStage;
          mbar_arrive_expect_tx(&sm.kv_full[stage], kStageBytes);
          tma_load_3d(kdst, mk, &sm.kv_full[stage], 0, ui.kvh, row);
          tma_load_3d(kdst + kKVBoxBytes, mk, &sm.kv_full[stage], 64, ui.kvh, row);
          tma_load_3d(vdst, mv, &sm.kv_full[stage], 0, ui.kvh, row);
          tma_load_3d(vdst + kKVBoxBytes, mv, &sm.kv_full[stage], 64, ui.kvh, row);
        }
        if (!ok) break;
        w.advance(p, hdr);
      }
      // make sure every copy this CTA issued has landed before the CTA can exit
      const long long nf = f;
      for (long long j = (nf > kStages ? nf - kStages : 0); j < nf; ++j) {
        const int stage = (int)(j % kStages);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&sm.kv_full[stage], (uint32_t)((j / kStages) & 1)) &&
               globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
      if (qn > 0) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&sm.q_full, (uint32_t)((qn - 1) & 1)) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer
    if (lane == 0) {
      SegWalk w;
      w.init(p, sm, hdr);
      long long f = 0;
      int seg = 0;
      bool ok = true;
      bool have_prev = false;
      long long prev_f = 0;
      bool prev_first = false;
      auto issue_pv = [&](long long pf, bool first) -> bool {
        const int stage = (int)(pf % kStages);
        const int bf = (int)(pf & 1);
        for (int h = 0; h < nh; ++h) {
          if (!mbar_wait_bounded(&sm.p_full[h][bf], (uint32_t)((pf >> 1) & 1), abort_flag)) {
            fail(kDetailWaitPFull);
            return false;
          }
          tc_fence_after();
          const uint32_t d_tm = tmem + (uint32_t)(kRowsPerHalf * h);
          const uint32_t p_tm = tmem + 256u + (uint32_t)(128 * h + 64 * bf);
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk) {
            const uint64_t bdesc = sdesc_sw128(sV + stage * kKBytesPerStage + kk * 2048, kKVBoxBytes, 1024);
            mma_ts(d_tm, p_tm + 8u * kk, bdesc, kIdescPV, (first && kk == 0) ? 0u : 1u);
          }
          tc_commit(&sm.pv_done[h][bf]);
        }
        tc_commit(&sm.kv_empty[stage]);
        return true;
      };
      while (ok && !w.done()) {
        int kb, ke;
        w.segment(kb, ke);
        if (!mbar_wait_bounded(&sm.q_full, (uint32_t)(seg & 1), abort_flag)) {
          fail(kDetailWaitQFull);
          ok = false;
          break;
        }
        tc_fence_after();
        for (int k = kb; k < ke; ++k, ++f) {
          const int stage = (int)(f % kStages);
          if (!mbar_wait_bounded(&sm.kv_full[stage], (uint32_t)((f / kStages) & 1), abort_flag)) {
            fail(kDetailWaitKvFull);
            ok = false;
            break;
          }
          tc_fence_after();
          const int bf = (int)(f & 1);
          for (int h = 0; h < nh; ++h) {
            const uint32_t d_tm = tmem + 256u + (uint32_t)(128 * h + 64 * bf);
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
              const uint32_t qa = sQ + (kk >> 2) * kQBytesPerDh + h * (kRowsPerHalf * 128) + (kk & 3) * 32;
              const uint32_t ka = sK + stage * kKBytesPerStage + (kk >> 2) * kKVBoxBytes + (kk & 3) * 32;
              mma_ss(d_tm, sdesc_sw128(qa, 16, 1024), sdesc_sw128(ka, 16, 1024), kIdescQK, kk > 0 ? 1u : 0u);
            }
            tc_commit(&sm.s_full[h][bf]);
          }
          if (k == ke - 1) tc_commit(&sm.q_empty);
          if (have_prev && !issue_pv(prev_f, prev_first)) {
            ok = false;
            break;
          }
          have_prev = true;
          prev_f = f;
          prev_first = (k == kb);
        }
        if (!ok) break;
        ++seg;
        w.advance(p, hdr);
      }
      if (ok && have_prev) issue_pv(prev_f, prev_first);
    }
  } else if (warp >= 4 && (warp - 4) / 4 < nh) {
    // ======================= softmax + epilogue, half h
    const int h = (warp - 4) / 4;
    const int t = tid - 128 - 128 * h;             // 0..127: TMEM lane and row within the half
    const int row = kRowsPerHalf * h + t;          // row within the unit's tile
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_tm0 = tmem + lane_off + 256u + (uint32_t)(128 * h);
    const uint32_t o_tm = tmem + lane_off + (uint32_t)(kRowsPerHalf * h);
    const float sc = p.scale_log2;
    float* partials = reinterpret_cast<float*>(p.ws + p.off_partials);
    float* plse = reinterpret_cast<float*>(p.ws + p.off_lse);
    SegWalk w;
    w.init(p, sm, hdr);
    long long f = 0;
    bool ok = true;
    while (ok && !w.done()) {
      int kb, ke;
      w.segment(kb, ke);
      const UnitInfo ui = w.ui;
      float m_used = -INFINITY, l = 0.f;
      for (int k = kb; k < ke; ++k, ++f) {
        const int bf = (int)(f & 1);
        const int valid = (k < ui.nctx) ? min(kTile, ui.L - k * kTile) : p.S;
        if (!mbar_wait_bounded(&sm.s_full[h][bf], (uint32_t)((f >> 1) & 1), abort_flag)) {
          fail(kDetailWaitSFull);
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld32(s_tm0 + 64u * bf, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(s_tm0 + 64u * bf + 32u, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_wait_ld();
        // row maximum of the raw scores (the scale is positive, so it commutes with max)
        float mt = -INFINITY;
        if (valid >= kTile) {
#pragma unroll
          for (int j = 0; j < 64; ++j) mt = fmaxf(mt, __uint_as_float(sr[j]));
        } else {
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            if (j >= valid) sr[j] = __float_as_uint(-INFINITY);
            mt = fmaxf(mt, __uint_as_float(sr[j]));
          }
        }
        mt *= sc;
        const bool first = (k == kb);
        bool resc = false;
        float m_new = m_used;
        if (first) {
          m_new = mt;
        } else if (mt > m_used + 8.0f) {
          m_new = mt;
          resc = true;
        }
        const float factor = resc ? ex2(m_used - m_new) : 1.0f;
        uint32_t pk[32];
        float psum0 = 0.f, psum1 = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float p0 = ex2(fmaf(__uint_as_float(sr[2 * j]), sc, -m_new));
          const float p1 = ex2(fmaf(__uint_as_float(sr[2 * j + 1]), sc, -m_new));
          psum0 += p0;
          psum1 += p1;
          pk[j] = pack_bf16x2(p0, p1);
        }
        l = l * factor + (psum0 + psum1);
        tmem_st32(s_tm0 + 64u * bf, pk);
        if (resc) {
          // O holds the sum up to tile f-1: wait for that PV product, then rescale it
          const long long pf = f - 1;
          if (!mbar_wait_bounded(&sm.pv_done[h][pf & 1], (uint32_t)((pf >> 1) & 1), abort_flag)) {
            fail(kDetailWaitPvDone);
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int cb = 0; cb < kD / 32; ++cb) {
            uint32_t orr[32];
            tmem_ld32(o_tm + 32u * cb, orr);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) orr[j] = __float_as_uint(__uint_as_float(orr[j]) * factor);
            tmem_st32(o_tm + 32u * cb, orr);
          }
        }
        tmem_wait_st();
        if (h == 0 && k < ui.nctx && valid < kTile) {
          // Rows past the end of the context hold whatever the caller's slab or page holds
          // there; P is 0 for them, but 0 * NaN would still poison O, so zero those V rows
          // before the PV product reads them (PV of half 1 is issued after half 0's).
          const int stage = (int)(f % kStages);
          uint8_t* vbase = smem + kSmemV + stage * kKBytesPerStage;
          const int chunks_per_box = (kTile - valid) * 8;   // 16-byte chunks
          for (int i = t; i < 2 * chunks_per_box; i += kRowsPerHalf) {
            const int box = i / chunks_per_box, r = i - box * chunks_per_box;
            *reinterpret_cast<uint4*>(vbase + box * kKVBoxBytes + (valid + r / 8) * 128 + (r % 8) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        m_used = m_new;
        tc_fence_before();
        mbar_arrive(&sm.p_full[h][bf]);
      }
      if (!ok) break;
      // ---- epilogue of the segment: wait for the last PV product, then O / l for this row
      const long long lf = f - 1;
      if (!mbar_wait_bounded(&sm.pv_done[h][lf & 1], (uint32_t)((lf >> 1) & 1), abort_flag)) {
        fail(kDetailWaitPvDone);
        ok = false;
        break;
      }
      tc_fence_after();
      const bool whole = (kb == 0) && (ke == ui.ntiles);
      const int s_cnt = min(p.s_per_tile, p.S - ui.qt * p.s_per_tile);
      const bool row_valid = row < p.G * s_cnt;
      const int s_idx = ui.qt * p.s_per_tile + row / p.G;
      const int hq = ui.kvh * p.G + row % p.G;
      const float inv_l = 1.0f / l;
      const float lse2 = m_used + log2f(l);
      const size_t slot = (size_t)w.u + (size_t)cta;   // unique per (unit, CTA) pair
      __nv_bfloat16* orow = p.out + (((size_t)ui.b * p.S + s_idx) * p.Hq + hq) * kD;
      float* prow = partials + (slot * 256 + row) * kD;
#pragma unroll 1
      for (int cb = 0; cb < kD / 32; ++cb) {
        uint32_t orr[32];
        tmem_ld32(o_tm + 32u * cb, orr);
        tmem_wait_ld();
        if (row_valid) {
          if (whole) {
            uint4* dst = reinterpret_cast<uint4*>(orow + cb * 32);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(orr[8 * q4 + 0]) * inv_l, __uint_as_float(orr[8 * q4 + 1]) * inv_l);
              v.y = pack_bf16x2(__uint_as_float(orr[8 * q4 + 2]) * inv_l, __uint_as_float(orr[8 * q4 + 3]) * inv_l);
              v.z = pack_bf16x2(__uint_as_float(orr[8 * q4 + 4]) * inv_l, __uint_as_float(orr[8 * q4 + 5]) * inv_l);
              v.w = pack_bf16x2(__uint_as_float(orr[8 * q4 + 6]) * inv_l, __uint_as_float(orr[8 * q4 + 7]) * inv_l);
              dst[q4] = v;
            }
          } else {
            float4* dst = reinterpret_cast<float4*>(prow + cb * 32);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              dst[q4] = make_float4(__uint_as_float(orr[4 * q4 + 0]) * inv_l, __uint_as_float(orr[4 * q4 + 1]) * inv_l,
                                    __uint_as_float(orr[4 * q4 + 2]) * inv_l, __uint_as_float(orr[4 * q4 + 3]) * inv_l);
          }
        }
      }
      if (row_valid) {
        if (whole) {
          if (p.lse) p.lse[((size_t)ui.b * p.Hq + hq) * p.S + s_idx] = lse2 * 0.69314718055994531f;
        } else {
          plse[slot * 256 + row] = lse2;
        }
      }
      w.advance(p, hdr);
    }
  }

  // ---- 3. teardown: all tensor-core work issued by the MMA thread completes before TMEM is
  // released (on the normal path it already has; on an abort path this drains it)
  if (warp == 1 && lane == 0) {
    tc_commit(&sm.drain);
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&sm.drain, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merges the partials of units cut between CTAs. One CTA per (unit, 32 query rows); a warp
// merges 4 rows, each lane 4 of the 128 dims, reading every contributor's row with coalesced
// 512-byte loads: O = sum_j 2^(lse_j - M) O_j / sum_j 2^(lse_j - M), M = max_j lse_j.
struct MergeParams {
  int32_t S, Hq, Hkv, G, qtiles, s_per_tile, units;
  __nv_bfloat16* out;
  float* lse;
  const uint8_t* ws;
  size_t off_meta, off_ustart, off_partials, off_lse;
};

__global__ void __launch_bounds__(256) attn_merge_kernel(const MergeParams p) {
  pdl_wait();
  const int u = blockIdx.x;
  const AttnMeta* meta = reinterpret_cast<const AttnMeta*>(p.ws + p.off_meta);
  const int32_t* ustart = reinterpret_cast<const int32_t*>(p.ws + p.off_ustart);
  const long long T = meta->total_tiles, Pe = meta->p_eff;
  if (T <= 0) return;
  const long long us = ustart[u], ue = ustart[u + 1];
  const long long c_lo = owner_cta(us, T, Pe), c_hi = owner_cta(ue - 1, T, Pe);
  if (c_lo == c_hi) return;   // a whole unit: the attention kernel wrote it
  const int qt = u % p.qtiles;
  const int bk = u / p.qtiles;
  const int kvh = bk % p.Hkv, b = bk / p.Hkv;
  const int s_cnt = min(p.s_per_tile, p.S - qt * p.s_per_tile);
  const int nrows = p.G * s_cnt;
  const float* partials = reinterpret_cast<const float*>(p.ws + p.off_partials);
  const float* plse = reinterpret_cast<const float*>(p.ws + p.off_lse);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = (int)(c_hi - c_lo + 1);
  for (int rr = 0; rr < 4; ++rr) {
    const int row = blockIdx.y * kMergeRows + warp * 4 + rr;
    if (row >= nrows) break;
    // per-contributor log2-sum-exp: lanes take contributors, then a warp max / sum
    float mx = -INFINITY;
    for (int j = lane; j < n; j += 32) mx = fmaxf(mx, plse[((size_t)u + (size_t)(c_lo + j)) * 256 + row]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float wsum = 0.f;
    for (int j0 = 0; j0 < n; j0 += 32) {
      const int j = j0 + lane;
      const float wl = (j < n) ? ex2(plse[((size_t)u + (size_t)(c_lo + j)) * 256 + row] - mx) : 0.f;
      float ws_part = wl;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ws_part += __shfl_xor_sync(0xffffffffu, ws_part, o);
      wsum += ws_part;
      const int cnt = min(32, n - j0);
      int jj = 0;
      for (; jj + 4 <= cnt; jj += 4) {
        float4 v[4];
        float wv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          wv[q] = __shfl_sync(0xffffffffu, wl, jj + q);
          const size_t sl = (size_t)u + (size_t)(c_lo + j0 + jj + q);
          v[q] = reinterpret_cast<const float4*>(partials + (sl * 256 + row) * kD)[lane];
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc.x = fmaf(wv[q], v[q].x, acc.x);
          acc.y = fmaf(wv[q], v[q].y, acc.y);
          acc.z = fmaf(wv[q], v[q].z, acc.z);
          acc.w = fmaf(wv[q], v[q].w, acc.w);
        }
      }
      for (; jj < cnt; ++jj) {
        const float wq = __shfl_sync(0xffffffffu, wl, jj);
        const size_t sl = (size_t)u + (size_t)(c_lo + j0 + jj);
        const float4 v = reinterpret_cast<const float4*>(partials + (sl * 256 + row) * kD)[lane];
        acc.x = fmaf(wq, v.x, acc.x);
        acc.y = fmaf(wq, v.y, acc.y);
        acc.z = fmaf(wq, v.z, acc.z);
        acc.w = fmaf(wq, v.w, acc.w);
      }
    }
    const float inv = 1.0f / wsum;
    const int s_idx = qt * p.s_per_tile + row / p.G;
    const int hq = kvh * p.G + row % p.G;
    __nv_bfloat16* orow = p.out + (((size_t)b * p.S + s_idx) * p.Hq + hq) * kD;
    uint2 o;
    o.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    o.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2*>(orow)[lane] = o;
    if (p.lse && lane == 0) p.lse[((size_t)b * p.Hq + hq) * p.S + s_idx] = (mx + log2f(wsum)) * 0.69314718055994531f;
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 3-D bf16 map: (d [contiguous], heads, rows), box (64, box_heads, box_rows), 128B swizzle.
bool make_map(CUtensorMap* m, const void* base, int heads, long long rows, int box_heads, int box_rows) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)heads, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)heads * kD * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Launch with the programmatic-stream-serialization attribute: the kernel may start while the
// previous kernel on the stream finishes; it reads no input before griddepcontrol.wait.
template <typename Kern, typename Params>
cudaError_t launch_pdl(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, const Params& prm) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, prm);
}

}  // namespace

bool attn_tc_supported(const tt_attn_args_t* a) {
  if (a->dtype != TT_BF16 || a->head_dim != kD) return false;
  const int G = a->num_q_heads / a->num_kv_heads;
  if (G > 256) return false;
  if (a->block_size > kTile) return false;
  if (a->page_table && (a->page_size % kTile) != 0) return false;
  // TMA needs 16-byte aligned bases
  const uintptr_t al = reinterpret_cast<uintptr_t>(a->q) | reinterpret_cast<uintptr_t>(a->k_blk) |
                       reinterpret_cast<uintptr_t>(a->v_blk) | reinterpret_cast<uintptr_t>(a->k_ctx) |
                       reinterpret_cast<uintptr_t>(a->v_ctx) | reinterpret_cast<uintptr_t>(a->out);
  if (al & 15) return false;
  return true;
}

AttnPlan attn_tc_plan(const tt_attn_args_t* a, int num_sms) {
  AttnPlan pl{};
  const int G = a->num_q_heads / a->num_kv_heads;
  const int S = a->block_size;
  pl.s_per_tile = std::min(S, 256 / G);
  pl.qtiles = (S + pl.s_per_tile - 1) / pl.s_per_tile;
  pl.units = a->batch * a->num_kv_heads * pl.qtiles;
  pl.grid = std::max(1, num_sms);
  pl.slots = (size_t)pl.units + (size_t)pl.grid;
  size_t off = kHeaderBytes;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = (off + bytes + 255) & ~size_t(255);
    return o;
  };
  pl.off_meta = take(sizeof(AttnMeta));
  pl.off_ustart = take(sizeof(int32_t) * ((size_t)pl.units + 1));
  pl.off_partials = take(sizeof(float) * pl.slots * 256 * kD);
  pl.off_lse = take(sizeof(float) * pl.slots * 256);
  pl.total = off;
  return pl;
}

int attn_tc_launch(const tt_attn_args_t* a, const AttnPlan& pl, void* ws, cudaStream_t stream) {
  TcParams p{};
  const int G = a->num_q_heads / a->num_kv_heads;
  const long long ctx_rows = a->page_table ? (long long)a->num_pages * a->page_size
                                           : (long long)a->batch * a->ctx_stride;
  if (!make_map(&p.tm_q, a->q, a->num_q_heads, (long long)a->batch * a->block_size, G, pl.s_per_tile))
    return TT_ERR_CUDA;
  if (!make_map(&p.tm_kc, a->k_ctx, a->num_kv_heads, std::max(1LL, ctx_rows), 1, kTile)) return TT_ERR_CUDA;
  if (!make_map(&p.tm_vc, a->v_ctx, a->num_kv_heads, std::max(1LL, ctx_rows), 1, kTile)) return TT_ERR_CUDA;
  if (!make_map(&p.tm_kb, a->k_blk, a->num_kv_heads, (long long)a->batch * a->block_size, 1, kTile))
    return TT_ERR_CUDA;
  if (!make_map(&p.tm_vb, a->v_blk, a->num_kv_heads, (long long)a->batch * a->block_size, 1, kTile))
    return TT_ERR_CUDA;
  p.ctx_lens = a->ctx_lens;
  p.page_table = a->page_table;
  p.B = a->batch;
  p.S = a->block_size;
  p.Hq = a->num_q_heads;
  p.Hkv = a->num_kv_heads;
  p.G = G;
  p.qtiles = pl.qtiles;
  p.s_per_tile = pl.s_per_tile;
  p.units = pl.units;
  p.page_size = a->page_size;
  p.max_pages = a->max_pages_per_seq;
  p.num_pages = a->num_pages;
  p.ctx_stride = a->ctx_stride;
  p.paged = a->page_table ? 1 : 0;
  p.scale_log2 = a->softmax_scale * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16*>(a->out);
  p.lse = a->lse;
  p.ws = static_cast<uint8_t*>(ws);
  p.off_meta = pl.off_meta;
  p.off_ustart = pl.off_ustart;
  p.off_partials = pl.off_partials;
  p.off_lse = pl.off_lse;
  // the shared-memory opt-in is per device; set it once so no attribute call happens while a
  // caller captures the stream into a CUDA graph
  static unsigned long long attr_done = 0;   // bit per device ordinal (< 64)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TT_ERR_CUDA;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(__atomic_load_n(&attr_done, __ATOMIC_ACQUIRE) & bit)) {
    if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) !=
        cudaSuccess)
      return TT_ERR_CUDA;
    __atomic_fetch_or(&attr_done, bit, __ATOMIC_ACQ_REL);
  }
  if (launch_pdl(attn_tc_kernel, dim3(pl.grid), dim3(kThreads), kSmemBytes, stream, p) != cudaSuccess)
    return TT_ERR_CUDA;
  MergeParams mp{};
  mp.S = p.S;
  mp.Hq = p.Hq;
  mp.Hkv = p.Hkv;
  mp.G = G;
  mp.qtiles = pl.qtiles;
  mp.s_per_tile = pl.s_per_tile;
  mp.units = pl.units;
  mp.out = p.out;
  mp.lse = p.lse;
  mp.ws = p.ws;
  mp.off_meta = pl.off_meta;
  mp.off_ustart = pl.off_ustart;
  mp.off_partials = pl.off_partials;
  mp.off_lse = pl.off_lse;
  const int M = G * pl.s_per_tile;
  const dim3 mgrid(pl.units, (M + kMergeRows - 1) / kMergeRows);
  if (launch_pdl(attn_merge_kernel, mgrid, dim3(256), 0, stream, mp) != cudaSuccess) return TT_ERR_CUDA;
  return TT_OK;
}

}  // namespace tt
