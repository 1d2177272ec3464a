// Eq. (1) of "Nemotron-TwoTower: Diffusion Language Modeling with Pretrained AR Context"
// (§2.1 "Bidirectional attention") for bf16 tensors on the sm_100a tensor cores.
//
// Work decomposition. A "group" is (sequence b, kv head): its keys are ceil(L_b/128) context
// tiles of 128 tokens followed by one tile holding the S block tokens. Its query rows are the
// G query heads of the kv head times the S block positions, packed as rows m = s * G + g and cut
// into "query tiles" of at most 128 rows (one tcgen05 M=128 MMA). nq = number of query tiles per
// group. A CTA holds two query tiles of a group (one for odd nq's last CTA), so the CTAs form
// teams of ceil(nq / 2); all groups' key tiles are laid end to end and cut into ranges, one per
// team, computed on the device from ctx_lens (no host knowledge of the lengths): either
// Pe = min(teams, tiles) equal ranges (ragged contexts balance to within a tile), or, when that
// costs at most kSegPenaltyTiles more per team, ranges that never cross a group boundary (each
// group cut into near-equal chunks), which spares the teams a second segment. For the common
// G * S = 256 one CTA holds the whole group: every K/V tile is staged once per group. A CTA that
// holds a whole group writes its rows of the output directly; a group cut between teams leaves a
// normalised partial (O_j / l_j and the log2-sum-exp) per query tile, and a second, wide kernel
// merges them (flash-decoding combine), launched as a programmatic dependent.
//
// Inside a CTA (384 threads: warpgroup 0 load and MMA, warpgroups 1-2 softmax), two independent
// softmax streams, one per query tile:
//   warps 0, 2 TMA producers: warp 0 the CTA's query tiles of the group and the K tiles of 128
//              tokens (2-stage ring), warp 2 the V tiles (2-stage ring), so that neither ring
//              waits for the other (128B-swizzled boxes; no multicast)
//   warp 1     MMA issuer (one thread): for stream j, S_j = Q_j K^T (M=128, N=128, K=128, both
//              operands from shared memory) and O_j += P_j V (A = P_j from TMEM, B = V). Per key
//              tile it issues PV_0(f), QK_0(f+1), PV_1(f), QK_1(f+1): while stream 0 runs its
//              softmax on tile f+1 the tensor pipe works for stream 1, and the other way round
//   warps 4-7  softmax + epilogue of stream 0, warps 8-11 of stream 1: a thread owns one query
//              row (its TMEM lane; lane quadrant = warp % 4) and all 128 key columns of a tile,
//              so the row maximum and sum need no exchange between threads
// TMEM (512 columns): O_0 [0,128), O_1 [128,256), S_0 [256,384), S_1 [384,512); a thread writes
// its row's 128 P values (bf16 pairs) over the first 64 columns of its S, which the PV product
// reads as its A operand.
// The softmax works in the exp2 domain with the scale folded in and computes P against the
// running maximum; only when a tile's maximum exceeds it by more than 8 (P > 256) does the
// base move to the tile maximum, with O rescaled (exact: numerator and denominator share the
// stale maximum).
// Groups with a single query tile (G * S <= 128) run a second kernel, attn_tc1_kernel (namespace
// `one` below), which puts both softmax warpgroups on that one tile; so do groups of two query
// tiles (a team of two CTAs, one tile each) when the key tiles per SM, bounded from the context
// capacity, are few (decode-sized work, where its faster pipeline fill and the smaller merge win).
#include <cstdio>
#include <cuda.h>
#include <cudaTypedefs.h>

#include "tt_common.cuh"
#include "tt_internal.h"

namespace tt {

namespace {

constexpr int kD = 128;           // head dim handled by this kernel
constexpr int kTile = 128;        // keys per tile
constexpr int kKStages = 2;       // K ring depth
constexpr int kVStages = 2;       // V ring depth
constexpr bool kSplitProducers = true;   // V loads from their own thread (warp 2), K and Q from warp 0
constexpr int kRows = 128;        // query rows per query tile (one M=128 MMA)
constexpr int kStreams = 2;       // query tiles (softmax streams) per CTA
// warpgroup 0: warp 0 TMA, warp 1 MMA (warps 2-3 idle); warpgroups 1-2: one softmax stream each
constexpr int kThreads = 128 + kStreams * kRows;
// Registers are handed out per warpgroup: the block launches with kLaunchRegs per thread, then the
// producer warpgroup gives registers back and the two softmax warpgroups take them (the sum stays
// within the launch pool: 128 * 88 + 256 * 208 = 384 * 168).
constexpr int kLaunchRegs = 168, kProducerRegs = 88, kSoftmaxRegs = 208;
static_assert(128 * kProducerRegs + 2 * 128 * kSoftmaxRegs <= kThreads * kLaunchRegs, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 256;  // S_j at column kTmemS + 128 j, O_j at 128 j

constexpr uint32_t kQBytesPerDh = kRows * 128;                 // 128 rows x 128 B = 16 KB
constexpr uint32_t kQBytes = 2 * kQBytesPerDh;                 // 32 KB per query tile
constexpr uint32_t kKVBoxBytes = kTile * 128;                  // 128 rows x 128 B = 16 KB
constexpr uint32_t kKBytesPerStage = 2 * kKVBoxBytes;          // 32 KB (two 64-dim boxes)
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemK = kStreams * kQBytes;
constexpr uint32_t kSmemV = kSmemK + kKStages * kKBytesPerStage;
constexpr uint32_t kSmemBar = kSmemV + kVStages * kKBytesPerStage;
constexpr uint32_t kSmemBytes = kSmemBar + 1024 + 1024;        // barriers + alignment slack


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

// Workspace: header | meta | contributors[groups] | partials | lse
struct AttnMeta {
  long long total_tiles;
  long long p_eff;   // working teams
};

// A team whose tile range crosses a group boundary runs two segments and pays a second epilogue
// and pipeline refill, worth about this many tiles of the steady-state loop (measured on the decode
// workload). The group-aligned partition is taken when its longest range is at most this much
// above the uniform one's.
constexpr long long kSegPenaltyTiles = 2;

// Groups of two query tiles take the one-tile kernel when the key tiles (bounded from the context
// capacity) are at most this many per SM.
constexpr long long kOneTileMaxTilesPerSm = 32;

struct TcParams {
  CUtensorMap tm_q, tm_kc, tm_vc, tm_kb, tm_vb;
  const int32_t* ctx_lens;
  const int32_t* page_table;
  int32_t B, S, Hq, Hkv, G;
  int32_t nq, nq2, s_per_tile, groups, teams;   // nq2 = CTAs per team = ceil(nq / 2)
  int32_t page_size, max_pages, num_pages, ctx_stride, paged;
  float scale_log2;   // softmax_scale * log2(e)
  __nv_bfloat16* out;
  float* lse;
  uint8_t* ws;
  size_t off_meta, off_crange, off_partials, off_lse;
  const int32_t* skip_if;
};

struct Smem {
  uint64_t q_full, q_empty;
  uint64_t k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[kStreams];   // S_j = Q_j K^T of the current tile is in TMEM
  uint64_t p_full[kStreams];   // P_j of the current tile is in TMEM (and O_j rescaled)
  uint64_t o_full[kStreams];   // O_j of the segment is complete
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  long long range_begin, range_end, total_tiles, p_eff;
  int u0;
  long long u0_start;
};
static_assert(sizeof(Smem) <= 1024, "barrier block");

struct GroupInfo {
  int b, kvh, L, nctx, ntiles;
};

__device__ __forceinline__ int clamp_len(const TcParams& p, int b, bool report, WsHeader* hdr) {
  int L = p.ctx_lens[b];
  if (L < 0) {
    if (report) report_error(hdr, TT_ERR_DEVICE, kDetailNegativeLen);
    L = 0;
  }
  const int cap = p.paged ? p.max_pages * p.page_size : p.ctx_stride;
  if (L > cap) {
    if (report) report_error(hdr, TT_ERR_DEVICE, kDetailCtxTooLong);
    L = cap;
  }
  return L;
}

__device__ __forceinline__ GroupInfo group_info(const TcParams& p, int g, bool report, WsHeader* hdr) {
  GroupInfo gi;
  gi.kvh = g % p.Hkv;
  gi.b = g / p.Hkv;
  gi.L = clamp_len(p, gi.b, report, hdr);
  gi.nctx = (gi.L + kTile - 1) / kTile;
  gi.ntiles = gi.nctx + 1;
  return gi;
}

// Walks the groups overlapping this team's tile range, one segment (a maximal run of tiles of one
// group) at a time. Every role runs its own copy; all copies see the same sequence.
struct SegWalk {
  int u;
  long long ustart;
  long long g, gend;
  GroupInfo gi;
  template <class Sm>
  __device__ void init(const TcParams& p, const Sm& sm, WsHeader* hdr) {
    u = sm.u0;
    ustart = sm.u0_start;
    g = sm.range_begin;
    gend = sm.range_end;
    gi = group_info(p, u, false, hdr);
  }
  __device__ bool done() const { return g >= gend; }
  // tiles [kb, ke) of group gi in the current segment
  __device__ void segment(int& kb, int& ke) const {
    kb = (int)(g - ustart);
    const long long uend = ustart + gi.ntiles;
    ke = (int)((uend < gend ? uend : gend) - ustart);
  }
  __device__ void advance(const TcParams& p, WsHeader* hdr) {
    int kb, ke;
    segment(kb, ke);
    g = ustart + ke;
    if (ke == gi.ntiles && g < gend) {
      ustart += gi.ntiles;
      ++u;
      gi = group_info(p, u, false, hdr);
    }
  }
};

// floor(a / b) for 0 <= a, 1 <= b, a + b < 2^53, through one double division (a 64-bit integer
// division is a long instruction sequence): a and b are exact in double, and a/b = q + r/b lies at
// least 1/b below q + 1, more than the division's rounding error (q + 1) 2^-53 when (q + 1) b < 2^53.
__device__ __forceinline__ long long floor_div(long long a, long long b) {
  return (long long)floor((double)a / (double)b);
}

// Team owning global tile t when T tiles are cut into P <= T ranges [c*T/P, (c+1)*T/P).
__device__ __forceinline__ long long owner_team(long long t, long long T, long long P) {
  return floor_div((t + 1) * P - 1, T);
}

// Warp 0 of every CTA: this team's tile range [range_begin, range_end) and the group where it
// starts, written to the CTA's shared block; CTA 0 also records, per group, the teams that hold its
// partials (for the merge kernel).
template <class Sm>
__device__ void partition_tiles(const TcParams& p, Sm& sm, int team, int lane, WsHeader* hdr) {
  // 32-bit arithmetic where the values allow it: 64-bit division is a long instruction
  // sequence, and this warp's chain of them sits before the first load
  auto wsum = [](uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
  };
  long long T = 0;
  int nmax = 0;
  int n_first = 0;   // this lane's group in the first 32 (kept: one read of ctx_lens for those)
  for (int base = 0; base < p.groups; base += 32) {
    const int u = base + lane;
    int n = 0;
    if (u < p.groups) n = group_info(p, u, blockIdx.x == 0, hdr).ntiles;
    if (base == 0) n_first = n;
    nmax = max(nmax, n);
    T += wsum((uint32_t)n);   // a group has fewer than 2^24 tiles (int32 lengths)
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) nmax = max(nmax, __shfl_xor_sync(0xffffffffu, nmax, o));
  auto ntiles_of = [&](int base, int u) -> int {
    return (u < p.groups) ? (base == 0 ? n_first : group_info(p, u, false, hdr).ntiles) : 0;
  };
  // with fewer tiles than teams only the first T teams work (one tile each), so every working
  // team owns a non-empty range and the teams of a group are consecutive
  const long long Pu = T < p.teams ? T : p.teams;
  uint32_t t_al = 0;   // chunk bound of the group-aligned partition; 0 = uniform
  if (T > 0 && T < (1LL << 31) && p.groups <= p.teams) {
    const uint32_t T32 = (uint32_t)T, teams32 = (uint32_t)p.teams, Pu32 = (uint32_t)Pu;
    // candidates t in [ceil(T/teams), ceil(T/Pu) + kSegPenaltyTiles], at most kSegPenaltyTiles + 1
    // of them (ceil(T/Pu) = ceil(T/teams) when Pu = teams, and both are 1 when Pu = T < teams):
    // sum_u ceil(n_u / t) for all of them in one pass, independent divisions side by side
    const uint32_t lo = (T32 - 1) / teams32 + 1;
    uint32_t hi = (T32 - 1) / Pu32 + 1 + (uint32_t)kSegPenaltyTiles;
    if (hi > (uint32_t)nmax) hi = (uint32_t)nmax;
    constexpr int kCand = (int)kSegPenaltyTiles + 1;
    uint32_t cnt[kCand];
#pragma unroll
    for (int k = 0; k < kCand; ++k) cnt[k] = 0;
    for (int base = 0; base < p.groups; base += 32) {
      const uint32_t n = (uint32_t)ntiles_of(base, base + lane);
#pragma unroll
      for (int k = 0; k < kCand; ++k) cnt[k] += (n + lo + k - 1) / (lo + k);
    }
#pragma unroll
    for (int k = 0; k < kCand; ++k) cnt[k] = wsum(cnt[k]);
    // the smallest feasible candidate (the count does not increase with t)
#pragma unroll
    for (int k = kCand - 1; k >= 0; --k)
      if (lo + k <= hi && cnt[k] <= teams32) t_al = lo + k;
  }
  const bool aligned = t_al > 0;
  long long rb = T, re = T;
  if (!aligned && team < Pu) {
    rb = floor_div(team * T, Pu);
    re = floor_div((team + 1) * T, Pu);
  }
  long long acc = 0, cacc = 0;
  int u0 = -1;
  long long u0s = 0;
  int2* crange_out = reinterpret_cast<int2*>(p.ws + p.off_crange);
  const bool record = (blockIdx.x == 0);
  for (int base = 0; base < p.groups && (u0 < 0 || record); base += 32) {
    const int u = base + lane;
    const int n = ntiles_of(base, u);
    const int c = aligned ? (int)(((uint32_t)n + t_al - 1) / t_al) : 0;   // chunks (teams) of group u
    int incl = n, cincl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      const int z = __shfl_up_sync(0xffffffffu, cincl, o);
      if (lane >= o) {
        incl += y;
        cincl += z;
      }
    }
    const long long lo = acc + incl - n, hi = acc + incl;   // tiles of group u
    const long long c0 = cacc + cincl - c;                  // its first team (aligned)
    if (record && u < p.groups) {
      // n >= 1 (the block tile), so hi - 1 >= lo
      crange_out[u] = aligned ? make_int2((int)c0, (int)(c0 + c - 1))
                              : make_int2((int)owner_team(lo, T, Pu), (int)owner_team(hi - 1, T, Pu));
    }
    const bool mine = u < p.groups && (aligned ? (c0 <= team && team < c0 + c) : (lo <= rb && rb < hi));
    const unsigned hit = __ballot_sync(0xffffffffu, mine);
    if (hit && u0 < 0) {
      const int src = __ffs(hit) - 1;
      u0 = base + src;
      u0s = __shfl_sync(0xffffffffu, lo, src);
      const uint32_t nn = (uint32_t)__shfl_sync(0xffffffffu, n, src);
      const uint32_t cc = (uint32_t)__shfl_sync(0xffffffffu, c, src);
      const uint32_t j = (uint32_t)(team - __shfl_sync(0xffffffffu, c0, src));
      if (aligned) {
        // chunk j covers [j*nn/cc, (j+1)*nn/cc) of the group, from the quotient and remainder
        // of nn/cc (j*nn may not fit 32 bits; j*r < cc^2 does)
        const uint32_t q = nn / cc, r = nn - q * cc;
        rb = u0s + (long long)j * q + (j * r) / cc;
        re = u0s + (long long)(j + 1) * q + ((j + 1) * r) / cc;
      }
    }
    acc += __shfl_sync(0xffffffffu, incl, 31);
    cacc += __shfl_sync(0xffffffffu, cincl, 31);
  }
  if (lane == 0) {
    sm.total_tiles = T;
    sm.p_eff = aligned ? cacc : Pu;
    sm.range_begin = rb;
    sm.range_end = re;
    sm.u0 = u0;
    sm.u0_start = u0s;
    sm.abort_flag = 0;
    if (record) {
      AttnMeta* meta = reinterpret_cast<AttnMeta*>(p.ws + p.off_meta);
      meta->total_tiles = T;
      meta->p_eff = aligned ? cacc : Pu;
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem& sm = *reinterpret_cast<Smem*>(smem + kSmemBar);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(p.ws);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int team = blockIdx.x / p.nq2;
  const int qt0 = 2 * (blockIdx.x % p.nq2);              // this CTA's first query tile
  const int nstreams = (qt0 + 1 < p.nq) ? 2 : 1;         // query tiles it holds

  // ---- 0. prologue that touches no input: barriers, TMEM, tensor-map prefetch. With a
  // programmatic launch it overlaps the previous kernel; inputs are read after pdl_wait().
  if (warp == 0 && lane == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&sm.v_full[i], 1);
      mbar_init(&sm.v_empty[i], 1);
    }
    for (int j = 0; j < kStreams; ++j) {
      mbar_init(&sm.s_full[j], 1);
      mbar_init(&sm.p_full[j], kRows / 32);   // one arrival per softmax warp
      mbar_init(&sm.o_full[j], 1);
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
  if (skip_requested(p.skip_if)) {
    // early exit of a multi-step loop: nothing to do; release TMEM and leave
    __syncthreads();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(sm.tmem_base, kTmemCols);
    }
    return;
  }

  // ---- 1. this team's tile range and the group where it starts (warp 0); CTA 0 also records,
  // per group, the teams that hold its partials (for the merge kernel).
  // Two partitions of the T tiles (in group order) are considered. Uniform: team c takes
  // [c*T/P, (c+1)*T/P), which balances tiles but lets ranges cross group boundaries. Group-aligned
  // (possible when groups <= teams): each group u is cut into ceil(n_u / t) near-equal chunks for
  // the smallest t with sum_u ceil(n_u / t) <= teams, one chunk per team, so no team runs two
  // segments. The aligned one is used when t <= ceil(T/P) + kSegPenaltyTiles.
  if (warp == 0) partition_tiles(p, sm, team, lane, hdr);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;
  const bool has_work = team < p.teams && sm.range_begin < sm.range_end && sm.u0 >= 0;

  auto fail = [&](uint32_t detail) {
    report_error(hdr, TT_ERR_DEVICE_TIMEOUT, detail);
    *abort_flag = 1;
  };

  const uint32_t sQ = smem_u32(smem + kSmemQ);
  const uint32_t sK = smem_u32(smem + kSmemK);
  const uint32_t sV = smem_u32(smem + kSmemV);

  if (warp < 4) {
    setmaxnreg_dec<kProducerRegs>();
  if (!has_work) {
    // nothing to do (more teams than tiles, or a CTA beyond the last full team)
  } else if (warp == 0 || (kSplitProducers && warp == 2)) {
    // ======================= TMA producers: warp 0 loads the query tiles and the K ring, warp 2
    // the V ring (warp 0 both when kSplitProducers is off), so that neither ring waits for the other
    if (lane == 0) {
      const bool do_kq = (warp == 0);
      const bool do_v = (warp == 2) || !kSplitProducers;
      SegWalk w;
      w.init(p, sm, hdr);
      long long f = 0;
      int qn = 0;
      bool ok = true;
      const uint32_t q_bytes = 2u * 128u * (uint32_t)p.G * (uint32_t)p.s_per_tile;   // one query tile
      while (ok && !w.done()) {
        int kb, ke;
        w.segment(kb, ke);
        const GroupInfo& gi = w.gi;
        if (do_kq) {
          if (qn > 0 && !mbar_wait_bounded(&sm.q_empty, (qn - 1) & 1, abort_flag)) {
            fail(kDetailWaitQEmpty);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.q_full, q_bytes * (uint32_t)nstreams);
          for (int j = 0; j < nstreams; ++j) {
            const int qrow = gi.b * p.S + (qt0 + j) * p.s_per_tile;
            uint8_t* qdst = smem + kSmemQ + j * kQBytes;
            tma_load_3d(qdst, &p.tm_q, &sm.q_full, 0, gi.kvh * p.G, qrow);
            tma_load_3d(qdst + kQBytesPerDh, &p.tm_q, &sm.q_full, 64, gi.kvh * p.G, qrow);
          }
          ++qn;
        }
        for (int k = kb; k < ke; ++k, ++f) {
          const CUtensorMap* mk;
          const CUtensorMap* mv;
          int row;
          if (k < gi.nctx) {
            const int t0 = k * kTile;
            if (p.paged) {
              int pg = p.page_table[(size_t)gi.b * p.max_pages + t0 / p.page_size];
              if (pg < 0 || pg >= p.num_pages) {
                report_error(hdr, TT_ERR_DEVICE, kDetailBadPage);
                pg = 0;   // read a valid page instead; the result is unspecified, the error is set
              }
              row = pg * p.page_size + t0 % p.page_size;
            } else {
              row = gi.b * p.ctx_stride + t0;
            }
            mk = &p.tm_kc;
            mv = &p.tm_vc;
          } else {
            row = gi.b * p.S;
            mk = &p.tm_kb;
            mv = &p.tm_vb;
          }
          if (do_kq) {
            // K of a stage is free once both streams' QK^T have read it
            const int ks = (int)(f % kKStages);
            const uint32_t kround = (uint32_t)(f / kKStages);
            if (kround > 0 && !mbar_wait_bounded(&sm.k_empty[ks], (kround - 1) & 1, abort_flag)) {
              fail(kDetailWaitKvEmpty);
              ok = false;
              break;
            }
            uint8_t* kdst = smem + kSmemK + ks * kKBytesPerStage;
            mbar_arrive_expect_tx(&sm.k_full[ks], kKBytesPerStage);
            tma_load_3d(kdst, mk, &sm.k_full[ks], 0, gi.kvh, row);
            tma_load_3d(kdst + kKVBoxBytes, mk, &sm.k_full[ks], 64, gi.kvh, row);
          }
          if (do_v) {
            // V of a stage is free once both streams' PV have read it
            const int vs = (int)(f % kVStages);
            const uint32_t vround = (uint32_t)(f / kVStages);
            if (vround > 0 && !mbar_wait_bounded(&sm.v_empty[vs], (vround - 1) & 1, abort_flag)) {
              fail(kDetailWaitKvEmpty);
              ok = false;
              break;
            }
            uint8_t* vdst = smem + kSmemV + vs * kKBytesPerStage;
            mbar_arrive_expect_tx(&sm.v_full[vs], kKBytesPerStage);
            tma_load_3d(vdst, mv, &sm.v_full[vs], 0, gi.kvh, row);
            tma_load_3d(vdst + kKVBoxBytes, mv, &sm.v_full[vs], 64, gi.kvh, row);
          }
        }
        if (!ok) break;
        w.advance(p, hdr);
      }
      // make sure every copy this thread issued has landed before the CTA can exit
      const long long nf = f;
      const uint64_t t0 = globaltimer_ns();
      if (do_kq) {
        for (long long jj = (nf > kKStages ? nf - kKStages : 0); jj < nf; ++jj)
          while (!mbar_try_wait(&sm.k_full[jj % kKStages], (uint32_t)((jj / kKStages) & 1)) &&
                 globaltimer_ns() - t0 < kWaitLimitNs) {
          }
        if (qn > 0)
          while (!mbar_try_wait(&sm.q_full, (uint32_t)((qn - 1) & 1)) && globaltimer_ns() - t0 < kWaitLimitNs) {
          }
      }
      if (do_v) {
        for (long long jj = (nf > kVStages ? nf - kVStages : 0); jj < nf; ++jj)
          while (!mbar_try_wait(&sm.v_full[jj % kVStages], (uint32_t)((jj / kVStages) & 1)) &&
                 globaltimer_ns() - t0 < kWaitLimitNs) {
          }
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer
    if (lane == 0) {
      SegWalk w;
      w.init(p, sm, hdr);
      // descriptor bases; per-MMA descriptors add constant offsets to the start-address field
      // (bits 0..13, 16-byte units), which shared-memory addresses below 256 KB never carry out of
      const uint64_t dq0 = sdesc_sw128(sQ, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(sK, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(sV, kKVBoxBytes, 1024);
      long long f = 0;
      int seg = 0;
      bool ok = true;
      // S_j = Q_j K^T for tile ff
      auto qk = [&](int j, long long ff) {
        const int stage = (int)(ff % kKStages);
        const uint32_t d_tm = tmem + kTmemS + 128u * (uint32_t)j;
        const uint64_t kd = dk0 + (uint64_t)((stage * kKBytesPerStage) >> 4);
        const uint64_t qd = dq0 + (uint64_t)((j * kQBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off_q = ((kk >> 2) * kQBytesPerDh + (kk & 3) * 32) >> 4;
          const uint32_t off_k = ((kk >> 2) * kKVBoxBytes + (kk & 3) * 32) >> 4;
          mma_ss(d_tm, qd + off_q, kd + off_k, kIdescQK, kk > 0 ? 1u : 0u);
        }
        tc_commit(&sm.s_full[j]);
      };
      // O_j (+)= P_j V for tile pf; P_j is in TMEM over the first 64 columns of S_j (keys 2c, 2c+1
      // in column c)
      auto pv = [&](int j, long long pf, bool first) {
        const int stage = (int)(pf % kVStages);
        const uint32_t p_tm = tmem + kTmemS + 128u * (uint32_t)j;
        const uint32_t o_tm = tmem + 128u * (uint32_t)j;
        const uint64_t vd = dv0 + (uint64_t)((stage * kKBytesPerStage) >> 4);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          mma_ts(o_tm, p_tm + 8u * (uint32_t)kk, vd + (uint64_t)((kk * 2048) >> 4), kIdescPV,
                 (first && kk == 0) ? 0u : 1u);
      };
      while (ok && !w.done()) {
        int kb, ke;
        w.segment(kb, ke);
        if (!mbar_wait_bounded(&sm.q_full, (uint32_t)(seg & 1), abort_flag)) {
          fail(kDetailWaitQFull);
          break;
        }
        // the segment's first tile: both streams' scores
        if (!mbar_wait_bounded(&sm.k_full[f % kKStages], (uint32_t)((f / kKStages) & 1), abort_flag)) {
          fail(kDetailWaitKvFull);
          break;
        }
        tc_fence_after();
        for (int j = 0; j < nstreams; ++j) qk(j, f);
        tc_commit(&sm.k_empty[f % kKStages]);
        if (ke - kb == 1) tc_commit(&sm.q_empty);
        for (int k = kb; k < ke && ok; ++k, ++f) {
          const bool first = (k == kb), last = (k == ke - 1);
          const int stage = (int)(f % kVStages);
          if (!mbar_wait_bounded(&sm.v_full[stage], (uint32_t)((f / kVStages) & 1), abort_flag)) {
            fail(kDetailWaitKvFull);
            ok = false;
            break;
          }
          for (int j = 0; j < nstreams; ++j) {
            // P_j of tile f written (and O_j rescaled) by stream j's softmax
            if (!mbar_wait_bounded(&sm.p_full[j], (uint32_t)(f & 1), abort_flag)) {
              fail(kDetailWaitPFull);
              ok = false;
              break;
            }
            tc_fence_after();
            pv(j, f, first);
            if (last) {
              tc_commit(&sm.o_full[j]);
            } else {
              // S_j is free again: P_j(f) is read by the PV just issued, which runs first
              const int nstage = (int)((f + 1) % kKStages);
              if (j == 0) {
                if (!mbar_wait_bounded(&sm.k_full[nstage], (uint32_t)(((f + 1) / kKStages) & 1), abort_flag)) {
                  fail(kDetailWaitKvFull);
                  ok = false;
                  break;
                }
                tc_fence_after();
              }
              qk(j, f + 1);
              if (j == nstreams - 1) {
                tc_commit(&sm.k_empty[nstage]);
                if (k + 1 == ke - 1) tc_commit(&sm.q_empty);
              }
            }
          }
          if (!ok) break;
          tc_commit(&sm.v_empty[stage]);
        }
        if (!ok) break;
        ++seg;
        w.advance(p, hdr);
      }
    }
  }
  } else {
    setmaxnreg_inc<kSoftmaxRegs>();
    // ======================= softmax + epilogue (stream j = warps 4-7 / 8-11)
    const int j = (warp - 4) >> 2;
    if (has_work && j < nstreams) {
      const int t = 32 * (warp & 3) + lane;   // TMEM lane quadrant warp % 4 -> query row t
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      const uint32_t s_tm = tmem + lane_off + kTmemS + 128u * (uint32_t)j;
      const uint32_t o_tm = tmem + lane_off + 128u * (uint32_t)j;
      const int qt = qt0 + j;
      const int s_cnt = min(p.s_per_tile, p.S - qt * p.s_per_tile);   // block positions of this query tile
      const int nrows = p.G * s_cnt;                                   // valid query rows (<= 128)
      const float sc = p.scale_log2;
      float* partials = reinterpret_cast<float*>(p.ws + p.off_partials);
      float* plse = reinterpret_cast<float*>(p.ws + p.off_lse);
      SegWalk w;
      w.init(p, sm, hdr);
      long long f = 0;
      int nseg = 0;
      bool ok = true;
      while (ok && !w.done()) {
        int kb, ke;
        w.segment(kb, ke);
        const GroupInfo gi = w.gi;
        float m_used = -INFINITY, l = 0.f;
        for (int k = kb; k < ke; ++k, ++f) {
          const int valid = (k < gi.nctx) ? min(kTile, gi.L - k * kTile) : p.S;
          if (!mbar_wait_bounded(&sm.s_full[j], (uint32_t)(f & 1), abort_flag)) {
            fail(kDetailWaitSFull);
            ok = false;
            break;
          }
          // The commit behind s_full also covers every earlier MMA of the issuing thread, so the
          // PV of the previous tile has completed: O_j may be read and rescaled below.
          __syncwarp();   // lanes leave the wait one by one; the tcgen05 accesses are warp-collective
          tc_fence_after();
          uint32_t sr[128];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            tmem_ld32(s_tm + 32u * (uint32_t)q, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * q]));
          tmem_wait_ld();
          if (valid < kTile) {
#pragma unroll
            for (int c = 0; c < kTile; ++c)
              if (c >= valid) sr[c] = __float_as_uint(-INFINITY);
          }
          // the row's tile maximum decides the exponent base: a segment's first tile uses it;
          // later tiles keep the running maximum m_used unless the tile exceeds it by more than 8
          // (P would exceed 256), in which case the base moves and O is rescaled
          float mx[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) mx[q] = __uint_as_float(sr[q]);
#pragma unroll
          for (int c = 4; c + 8 <= kTile; c += 8) {
#pragma unroll
            for (int q = 0; q < 4; ++q) mx[q] = fmax3(mx[q], __uint_as_float(sr[c + q]), __uint_as_float(sr[c + 4 + q]));
          }
          mx[0] = fmax3(mx[0], __uint_as_float(sr[kTile - 4]), __uint_as_float(sr[kTile - 3]));
          mx[1] = fmax3(mx[1], __uint_as_float(sr[kTile - 2]), __uint_as_float(sr[kTile - 1]));
          const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sc;
          const bool first = (k == kb);
          float m_new = m_used;
          bool resc = false;
          if (first) {
            m_new = mt;
          } else if (mt > m_used + 8.0f) {
            m_new = mt;
            resc = true;
          }
          // P = 2^(s * scale - base), written as bf16 pairs over the first 64 columns of S_j,
          // summed in fp32
          const uint64_t sc2 = pack_f32x2(sc, sc);
          const uint64_t nb2 = pack_f32x2(-m_new, -m_new);
          uint64_t acc2[2] = {pack_f32x2(0.f, 0.f), pack_f32x2(0.f, 0.f)};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t pk[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int c = 32 * q + 2 * jj;
              const uint64_t x2 = ffma_f32x2(pack_u32x2(sr[c], sr[c + 1]), sc2, nb2);
              const float p0 = ex2(lo_f32(x2)), p1 = ex2(hi_f32(x2));
              const uint64_t p2 = pack_f32x2(p0, p1);
              acc2[jj & 1] = fadd_f32x2(acc2[jj & 1], p2);
              pk[jj] = pack_bf16x2(p0, p1);
            }
            tmem_st16(s_tm + 16u * (uint32_t)q, pk);
          }
          const uint64_t acc = fadd_f32x2(acc2[0], acc2[1]);
          const float psum = lo_f32(acc) + hi_f32(acc);
          const float factor = resc ? ex2(m_used - m_new) : 1.0f;
          l = l * factor + psum;
          tmem_wait_st();
          if (!first && __any_sync(0xffffffffu, resc)) {
            // rows decide separately; the O accesses are warp-collective, so the warp rescales when
            // any of its rows needs it (factor is 1 for the others)
#pragma unroll 1
            for (int cb = 0; cb < 4; ++cb) {
              uint32_t orr[32];
              tmem_ld32(o_tm + 32u * (uint32_t)cb, orr);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * factor);
              tmem_st32(o_tm + 32u * (uint32_t)cb, orr);
            }
            tmem_wait_st();
          }
          if (j == 0 && k < gi.nctx && valid < kTile) {
            // Rows past the end of the context hold whatever the caller's slab or page holds
            // there; P is 0 for them, but 0 * NaN would still poison O, so zero those V rows
            // before the PV products (stream 0's runs first) read them. The V tile must have
            // landed first.
            const int stage = (int)(f % kVStages);
            if (!mbar_wait_bounded(&sm.v_full[stage], (uint32_t)((f / kVStages) & 1), abort_flag)) {
              fail(kDetailWaitKvFull);
              ok = false;
              break;
            }
            uint8_t* vbase = smem + kSmemV + stage * kKBytesPerStage;
            const int chunks_per_box = (kTile - valid) * 8;   // 16-byte chunks
            for (int i = t; i < 2 * chunks_per_box; i += kRows) {
              const int box = i / chunks_per_box, r = i - box * chunks_per_box;
              *reinterpret_cast<uint4*>(vbase + box * kKVBoxBytes + (valid + r / 8) * 128 + (r % 8) * 16) =
                  make_uint4(0u, 0u, 0u, 0u);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          }
          m_used = m_new;
          // every lane's TMEM stores (and O rescale) are complete and fenced before the warp's one
          // arrival hands P to the MMA thread
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.p_full[j]);
        }
        if (!ok) break;
        // ---- epilogue of the segment: wait for the last PV product, then O / l for the row
        if (!mbar_wait_bounded(&sm.o_full[j], (uint32_t)(nseg & 1), abort_flag)) {
          fail(kDetailWaitPvDone);
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        ++nseg;
        const bool whole = (kb == 0) && (ke == gi.ntiles);
        const bool row_valid = t < nrows;
        const int s_idx = qt * p.s_per_tile + t / p.G;
        const int hq = gi.kvh * p.G + t % p.G;
        const float inv_l = 1.0f / l;
        const float lse2 = m_used + log2f(l);
        // partial slot unique per (group, team, query tile)
        const size_t slot = ((size_t)w.u + (size_t)team) * (size_t)p.nq + (size_t)qt;
        __nv_bfloat16* orow = p.out + (((size_t)gi.b * p.S + s_idx) * p.Hq + hq) * kD;
        float* prow = partials + (slot * kRows + t) * kD;
#pragma unroll 1
        for (int cb = 0; cb < 4; ++cb) {
          uint32_t orr[32];
          tmem_ld32(o_tm + 32u * (uint32_t)cb, orr);
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
            if (p.lse) p.lse[((size_t)gi.b * p.Hq + hq) * p.S + s_idx] = lse2 * 0.69314718055994531f;
          } else {
            plse[slot * kRows + t] = lse2;
          }
        }
        w.advance(p, hdr);
      }
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

// ---------------------------------------------------------------------------------------------
// Groups with a single query tile (G * S <= 128, e.g. S <= 8 at G = 16): the two-stream kernel
// above would run one softmax stream per CTA and leave the other warpgroup idle. This kernel
// puts the tile's work on both: one query tile per CTA; the softmax split by key columns between
// the two warpgroups (a thread owns one query row and 64 of a tile's 128 columns; the row's two
// threads exchange their maxima once per tile and their sums once per segment through shared
// memory and a named barrier of the warp pair); three S buffers in TMEM (O [0,128), S at 128,
// 256, 384) so that the scores run three tiles ahead of the PV products, which the softmax of
// the next tile therefore never waits for; warp 3 issues the QK products and warp 1 the PV
// products (one thread each; a QK refills its S buffer once the PV that read P there has
// completed); warp 0 loads the query tile and a 3-stage K ring, warp 2 a 2-stage V ring. The
// partition of the key tiles, the segment walk, the output and the split-KV partials are those
// of the two-stream kernel.
namespace one {

constexpr int kKStages = 3;       // K ring depth (= kSBufs: a stage's QK completion is also its S)
constexpr int kVStages = 2;       // V ring depth
constexpr int kSBufs = 3;         // S buffers in TMEM: QK runs this many tiles ahead of PV
static_assert(kKStages == kSBufs, "k_empty[g % kSBufs] doubles as the S-ready barrier of tile g");
constexpr int kHalves = 2;        // softmax warpgroups, each 64 of a tile's 128 key columns
constexpr int kThreads = 128 + kHalves * kRows;
constexpr int kLaunchRegs = 168, kProducerRegs = 88, kSoftmaxRegs = 208;
static_assert(128 * kProducerRegs + 2 * 128 * kSoftmaxRegs <= kThreads * kLaunchRegs, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 128;  // O at columns [0, 128), S buffer b at kTmemS + 128 b
static_assert(kTmemS + 128 * kSBufs <= kTmemCols, "TMEM budget");
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemK = kQBytes;
constexpr uint32_t kSmemV = kSmemK + kKStages * kKBytesPerStage;
constexpr uint32_t kSmemBar = kSmemV + kVStages * kKBytesPerStage;
// the two halves' exchanges (row maxima per tile, row sums per segment): values and the warps'
// good flags, double-buffered by exchange parity
constexpr uint32_t kSmemX = kSmemBar + 1024;
constexpr uint32_t kXBytes = 2 * kHalves * kRows * 4 + 2 * kHalves * 4 * 4;
constexpr uint32_t kSmemBytes = kSmemX + kXBytes + 1024;       // + alignment slack

struct Smem {
  uint64_t q_full, q_empty;
  uint64_t k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  // k_empty[b] completes when the QK of a tile using K stage b = S buffer b has completed: the K
  // stage is free and the tile's S is ready (one phase per tile using b)
  uint64_t p_full[kSBufs];     // P of a tile is in S buffer b (and O rescaled): both halves' warps
  uint64_t pv_done[kSBufs];    // O += P V of a tile using S buffer b has completed
  uint64_t o_full;             // O of the segment is complete (one phase per segment)
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  long long range_begin, range_end, total_tiles, p_eff;
  int u0;
  long long u0_start;
};
static_assert(sizeof(Smem) <= 1024, "barrier block");

// Slot and phase parity of use n of an R-deep ring (a CTA's tile counters: n < 2^32), in 32-bit
// arithmetic (a 64-bit division is a long instruction sequence, and these sit in every tile's chain).
template <int R>
__device__ __forceinline__ int ring_slot(long long n) {
  return (int)((uint32_t)n % (uint32_t)R);
}
template <int R>
__device__ __forceinline__ uint32_t ring_phase(long long n) {
  return ((uint32_t)n / (uint32_t)R) & 1u;
}

__global__ void __launch_bounds__(kThreads, 1) attn_tc1_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem& sm = *reinterpret_cast<Smem*>(smem + kSmemBar);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(p.ws);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int team = blockIdx.x / p.nq;
  const int qt = blockIdx.x % p.nq;                      // this CTA's query tile

  // ---- 0. prologue that touches no input: barriers, TMEM, tensor-map prefetch. With a
  // programmatic launch it overlaps the previous kernel; inputs are read after pdl_wait().
  if (warp == 0 && lane == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&sm.v_full[i], 1);
      mbar_init(&sm.v_empty[i], 1);
    }
    for (int b = 0; b < kSBufs; ++b) {
      mbar_init(&sm.p_full[b], kHalves * kRows / 32);   // one arrival per softmax warp
      mbar_init(&sm.pv_done[b], 1);
    }
    mbar_init(&sm.o_full, 1);
    mbar_init(&sm.drain, 2);   // both MMA-issuing threads
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
  if (skip_requested(p.skip_if)) {
    // early exit of a multi-step loop: nothing to do; release TMEM and leave
    __syncthreads();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(sm.tmem_base, kTmemCols);
    }
    return;
  }

  // ---- 1. this team's tile range and the group where it starts (warp 0); CTA 0 also records,
  // per group, the teams that hold its partials (for the merge kernel).
  // Two partitions of the T tiles (in group order) are considered. Uniform: team c takes
  // [c*T/P, (c+1)*T/P), which balances tiles but lets ranges cross group boundaries. Group-aligned
  // (possible when groups <= teams): each group u is cut into ceil(n_u / t) near-equal chunks for
  // the smallest t with sum_u ceil(n_u / t) <= teams, one chunk per team, so no team runs two
  // segments. The aligned one is used when t <= ceil(T/P) + kSegPenaltyTiles.
  if (warp == 0) partition_tiles(p, sm, team, lane, hdr);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;
  const bool has_work = team < p.teams && sm.range_begin < sm.range_end && sm.u0 >= 0;

  auto fail = [&](uint32_t detail) {
    report_error(hdr, TT_ERR_DEVICE_TIMEOUT, detail);
    *abort_flag = 1;
  };

  const uint32_t sQ = smem_u32(smem + kSmemQ);
  const uint32_t sK = smem_u32(smem + kSmemK);
  const uint32_t sV = smem_u32(smem + kSmemV);

  if (warp < 4) {
    setmaxnreg_dec<kProducerRegs>();
  if (!has_work) {
    // nothing to do (more teams than tiles, or a CTA beyond the last full team)
  } else if (warp == 0 || warp == 2) {
    // ======================= TMA producers: warp 0 loads the query tiles and the K ring, warp 2
    // the V ring, so that neither ring waits for the other
    if (lane == 0) {
      const bool do_kq = (warp == 0);
      const bool do_v = (warp == 2);
      SegWalk w;
      w.init(p, sm, hdr);
      long long f = 0;
      int qn = 0;
      bool ok = true;
      const uint32_t q_bytes = 2u * 128u * (uint32_t)p.G * (uint32_t)p.s_per_tile;   // one query tile
      while (ok && !w.done()) {
        int kb, ke;
        w.segment(kb, ke);
        const GroupInfo& gi = w.gi;
        if (do_kq) {
          if (qn > 0 && !mbar_wait_bounded(&sm.q_empty, (qn - 1) & 1, abort_flag)) {
            fail(kDetailWaitQEmpty);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.q_full, q_bytes);
          const int qrow = gi.b * p.S + qt * p.s_per_tile;
          uint8_t* qdst = smem + kSmemQ;
          tma_load_3d(qdst, &p.tm_q, &sm.q_full, 0, gi.kvh * p.G, qrow);
          tma_load_3d(qdst + kQBytesPerDh, &p.tm_q, &sm.q_full, 64, gi.kvh * p.G, qrow);
          ++qn;
        }
        for (int k = kb; k < ke; ++k, ++f) {
          const CUtensorMap* mk;
          const CUtensorMap* mv;
          int row;
          if (k < gi.nctx) {
            const int t0 = k * kTile;
            if (p.paged) {
              int pg = p.page_table[(size_t)gi.b * p.max_pages + t0 / p.page_size];
              if (pg < 0 || pg >= p.num_pages) {
                report_error(hdr, TT_ERR_DEVICE, kDetailBadPage);
                pg = 0;   // read a valid page instead; the result is unspecified, the error is set
              }
              row = pg * p.page_size + t0 % p.page_size;
            } else {
              row = gi.b * p.ctx_stride + t0;
            }
            mk = &p.tm_kc;
            mv = &p.tm_vc;
          } else {
            row = gi.b * p.S;
            mk = &p.tm_kb;
            mv = &p.tm_vb;
          }
          if (do_kq) {
            // K of a stage is free once its QK^T has read it
            const int ks = ring_slot<kKStages>(f);
            const uint32_t kround = (uint32_t)f / (uint32_t)kKStages;
            if (kround > 0 && !mbar_wait_bounded(&sm.k_empty[ks], (kround - 1) & 1, abort_flag)) {
              fail(kDetailWaitKvEmpty);
              ok = false;
              break;
            }
            uint8_t* kdst = smem + kSmemK + ks * kKBytesPerStage;
            mbar_arrive_expect_tx(&sm.k_full[ks], kKBytesPerStage);
            tma_load_3d(kdst, mk, &sm.k_full[ks], 0, gi.kvh, row);
            tma_load_3d(kdst + kKVBoxBytes, mk, &sm.k_full[ks], 64, gi.kvh, row);
          }
          if (do_v) {
            // V of a stage is free once its PV has read it
            const int vs = ring_slot<kVStages>(f);
            const uint32_t vround = (uint32_t)f / (uint32_t)kVStages;
            if (vround > 0 && !mbar_wait_bounded(&sm.v_empty[vs], (vround - 1) & 1, abort_flag)) {
              fail(kDetailWaitKvEmpty);
              ok = false;
              break;
            }
            uint8_t* vdst = smem + kSmemV + vs * kKBytesPerStage;
            mbar_arrive_expect_tx(&sm.v_full[vs], kKBytesPerStage);
            tma_load_3d(vdst, mv, &sm.v_full[vs], 0, gi.kvh, row);
            tma_load_3d(vdst + kKVBoxBytes, mv, &sm.v_full[vs], 64, gi.kvh, row);
          }
        }
        if (!ok) break;
        w.advance(p, hdr);
      }
      // make sure every copy this thread issued has landed before the CTA can exit
      const long long nf = f;
      const uint64_t t0 = globaltimer_ns();
      if (do_kq) {
        for (long long jj = (nf > kKStages ? nf - kKStages : 0); jj < nf; ++jj)
          while (!mbar_try_wait(&sm.k_full[jj % kKStages], (uint32_t)((jj / kKStages) & 1)) &&
                 globaltimer_ns() - t0 < kWaitLimitNs) {
          }
        if (qn > 0)
          while (!mbar_try_wait(&sm.q_full, (uint32_t)((qn - 1) & 1)) && globaltimer_ns() - t0 < kWaitLimitNs) {
          }
      }
      if (do_v) {
        for (long long jj = (nf > kVStages ? nf - kVStages : 0); jj < nf; ++jj)
          while (!mbar_try_wait(&sm.v_full[jj % kVStages], (uint32_t)((jj / kVStages) & 1)) &&
                 globaltimer_ns() - t0 < kWaitLimitNs) {
          }
      }
    }
  } else if (warp == 1 || warp == 3) {
    // ======================= MMA issuers: warp 1 the PV products, warp 3 the QK products (one
    // thread each; each thread's products run in its issue order, the two threads' products
    // interleave on the tensor pipe)
    if (lane == 0) {
      SegWalk w;
      w.init(p, sm, hdr);
      // descriptor bases; per-MMA descriptors add constant offsets to the start-address field
      // (bits 0..13, 16-byte units), which shared-memory addresses below 256 KB never carry out of
      const uint64_t dq0 = sdesc_sw128(sQ, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(sK, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(sV, kKVBoxBytes, 1024);
      long long f = 0;   // tiles of this CTA so far (all segments)
      int seg = 0;
      bool ok = true;
      while (ok && !w.done()) {
        int kb, ke;
        w.segment(kb, ke);
        const long long fs = f, fe = f + (ke - kb);   // this segment's tiles [fs, fe)
        if (warp == 3) {
          // S(g) = Q K(g)^T into S buffer g % kSBufs. That buffer held P of tile g - kSBufs: wait
          // for its PV (pv_done is then exactly one phase behind: PV(g) needs this S first).
          if (!mbar_wait_bounded(&sm.q_full, (uint32_t)(seg & 1), abort_flag)) {
            fail(kDetailWaitQFull);
            break;
          }
          for (; f < fe; ++f) {
            const int b = ring_slot<kSBufs>(f);
            if (f >= kSBufs) {
              if (!mbar_wait_bounded(&sm.pv_done[b], ring_phase<kSBufs>(f - kSBufs), abort_flag)) {
                fail(kDetailWaitPvDone);
                ok = false;
                break;
              }
            }
            if (!mbar_wait_bounded(&sm.k_full[b], ring_phase<kKStages>(f), abort_flag)) {
              fail(kDetailWaitKvFull);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t d_tm = tmem + kTmemS + 128u * (uint32_t)b;
            const uint64_t kd = dk0 + (uint64_t)((b * kKBytesPerStage) >> 4);
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
              const uint32_t off_q = ((kk >> 2) * kQBytesPerDh + (kk & 3) * 32) >> 4;
              const uint32_t off_k = ((kk >> 2) * kKVBoxBytes + (kk & 3) * 32) >> 4;
              mma_ss(d_tm, dq0 + off_q, kd + off_k, kIdescQK, kk > 0 ? 1u : 0u);
            }
            tc_commit(&sm.k_empty[b]);   // K stage free, S of tile f ready
            if (f == fe - 1) tc_commit(&sm.q_empty);
          }
        } else {
          // O (+)= P(f) V(f); P is in TMEM over the first 64 columns of S buffer f % kSBufs (keys
          // 2c, 2c+1 in column c)
          for (; f < fe; ++f) {
            const int stage = ring_slot<kVStages>(f);
            const int b = ring_slot<kSBufs>(f);
            if (!mbar_wait_bounded(&sm.v_full[stage], ring_phase<kVStages>(f), abort_flag)) {
              fail(kDetailWaitKvFull);
              ok = false;
              break;
            }
            // P of tile f written (and O rescaled) by both halves of the softmax
            if (!mbar_wait_bounded(&sm.p_full[b], ring_phase<kSBufs>(f), abort_flag)) {
              fail(kDetailWaitPFull);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t p_tm = tmem + kTmemS + 128u * (uint32_t)b;
            const uint64_t vd = dv0 + (uint64_t)((stage * kKBytesPerStage) >> 4);
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk)
              mma_ts(tmem, p_tm + 8u * (uint32_t)kk, vd + (uint64_t)((kk * 2048) >> 4), kIdescPV,
                     (f == fs && kk == 0) ? 0u : 1u);
            tc_commit(&sm.pv_done[b]);
            tc_commit(&sm.v_empty[stage]);
            if (f == fe - 1) tc_commit(&sm.o_full);
          }
        }
        if (!ok) break;
        ++seg;
        w.advance(p, hdr);
      }
    }
  }
  } else {
    setmaxnreg_inc<kSoftmaxRegs>();
    // ======================= softmax + epilogue: warps 4-7 (half 0) and 8-11 (half 1). A thread
    // owns one query row (its TMEM lane; lane quadrant = warp % 4) and 64 of a tile's 128 key
    // columns; the two threads of a row (warps w and w + 4) exchange their maxima once per tile
    // and their sums once per segment through shared memory and a named barrier of the pair.
    // Leaving early: a failed bounded wait only marks the warp (good = false, error recorded,
    // later waits return at once) and the work goes on; the pair leaves together after its next
    // exchange, which carries both warps' marks, so neither is ever left alone at the barrier.
    const int h = (warp - 4) >> 2;            // column half
    const int quad = warp & 3;
    const int t = 32 * quad + lane;           // query row
    if (has_work) {
      const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
      const uint32_t o_tm = tmem + lane_off + 64u * (uint32_t)h;
      const int s_cnt = min(p.s_per_tile, p.S - qt * p.s_per_tile);   // block positions of this query tile
      const int nrows = p.G * s_cnt;                                   // valid query rows (<= 128)
      const float sc = p.scale_log2;
      float* partials = reinterpret_cast<float*>(p.ws + p.off_partials);
      float* plse = reinterpret_cast<float*>(p.ws + p.off_lse);
      float* xv = reinterpret_cast<float*>(smem + kSmemX);             // [exchange parity][half][row]
      int* xg = reinterpret_cast<int*>(xv + 2 * kHalves * kRows);      // [exchange parity][half][quadrant]
      uint32_t xph = 0;                                                // exchanges so far
      bool good = true;                                                // warp-uniform
      // a bounded wait that records a failure instead of leaving
      auto wait = [&](uint64_t* bar, uint32_t parity, uint32_t detail) {
        bool got = true;
        if (good) {
          got = mbar_wait_bounded(bar, parity, abort_flag);
          if (!got) fail(detail);
        }
        good = __all_sync(0xffffffffu, good && got);
      };
      // hands `v` to the row's other half and reads the other half's value into `other`; returns
      // whether both warps of the pair are still good (the same answer in both)
      auto exchange = [&](float v, float& other) -> bool {
        float* slot = xv + (xph & 1u) * kHalves * kRows;
        int* flg = xg + (xph & 1u) * kHalves * 4;
        ++xph;
        slot[h * kRows + t] = v;
        if (lane == 0) flg[h * 4 + quad] = good ? 1 : 0;
        named_barrier_sync(1 + quad, 64);
        other = slot[(1 - h) * kRows + t];
        return flg[(1 - h) * 4 + quad] != 0 && good;
      };
      SegWalk w;
      w.init(p, sm, hdr);
      long long f = 0;
      int nseg = 0;
      bool ok = true;
      while (ok && !w.done()) {
        int kb, ke;
        w.segment(kb, ke);
        const GroupInfo gi = w.gi;
        float m_used = -INFINITY, l = 0.f;   // running base; this half's running sum
        for (int k = kb; k < ke; ++k, ++f) {
          const int valid = (k < gi.nctx) ? min(kTile, gi.L - k * kTile) : p.S;
          const int b = ring_slot<kSBufs>(f);
          const uint32_t s_tm = tmem + lane_off + kTmemS + 128u * (uint32_t)b;
          wait(&sm.k_empty[b], ring_phase<kSBufs>(f), kDetailWaitSFull);
          // (after a failed wait the work below still runs, on whatever TMEM holds: its results
          // are discarded when the pair leaves at the exchange)
          __syncwarp();   // lanes leave the wait one by one; the tcgen05 accesses are warp-collective
          tc_fence_after();
          uint32_t sr[64];
          tmem_ld32(s_tm + 64u * (uint32_t)h, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
          tmem_ld32(s_tm + 64u * (uint32_t)h + 32u, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
          tmem_wait_ld();
          const int valid_h = valid - 64 * h;   // valid keys among this half's columns
          if (valid_h < 64) {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (c >= valid_h) sr[c] = __float_as_uint(-INFINITY);
          }
          float mx[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) mx[q] = __uint_as_float(sr[q]);
#pragma unroll
          for (int c = 4; c + 8 <= 64; c += 8) {
#pragma unroll
            for (int q = 0; q < 4; ++q) mx[q] = fmax3(mx[q], __uint_as_float(sr[c + q]), __uint_as_float(sr[c + 4 + q]));
          }
          mx[0] = fmax3(mx[0], __uint_as_float(sr[60]), __uint_as_float(sr[61]));
          mx[1] = fmax3(mx[1], __uint_as_float(sr[62]), __uint_as_float(sr[63]));
          const float mh = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sc;
          // the row's tile maximum (both halves) decides the exponent base: a segment's first tile
          // uses it; later tiles keep the running maximum m_used unless the tile exceeds it by more
          // than 8 (P would exceed 256), in which case the base moves and O is rescaled. Both
          // threads of a row see the same two values and take the same decision.
          float mo;
          if (!exchange(mh, mo)) {
            ok = false;
            break;
          }
          const float mt = fmaxf(mh, mo);
          const bool first = (k == kb);
          float m_new = m_used;
          bool resc = false;
          if (first) {
            m_new = mt;
          } else if (mt > m_used + 8.0f) {
            m_new = mt;
            resc = true;
          }
          // P = 2^(s * scale - base), written as bf16 pairs over columns [32 h, 32 h + 32) of the
          // S buffer (the other half's S columns there were read before the exchange), summed in fp32
          const uint32_t p_tm = s_tm + 32u * (uint32_t)h;
          const uint64_t sc2 = pack_f32x2(sc, sc);
          const uint64_t nb2 = pack_f32x2(-m_new, -m_new);
          uint64_t acc2[2] = {pack_f32x2(0.f, 0.f), pack_f32x2(0.f, 0.f)};
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint32_t pk[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int c = 32 * q + 2 * jj;
              const uint64_t x2 = ffma_f32x2(pack_u32x2(sr[c], sr[c + 1]), sc2, nb2);
              const float p0 = ex2(lo_f32(x2)), p1 = ex2(hi_f32(x2));
              acc2[jj & 1] = fadd_f32x2(acc2[jj & 1], pack_f32x2(p0, p1));
              pk[jj] = pack_bf16x2(p0, p1);
            }
            tmem_st16(p_tm + 16u * (uint32_t)q, pk);
          }
          const uint64_t acc = fadd_f32x2(acc2[0], acc2[1]);
          const float psum = lo_f32(acc) + hi_f32(acc);
          const float factor = resc ? ex2(m_used - m_new) : 1.0f;
          l = l * factor + psum;
          tmem_wait_st();
          if (!first && __any_sync(0xffffffffu, resc)) {
            // O holds the products up to tile f - 1, the last of which may still be running: wait
            // for it (the S of this tile came from a QK issued after the PV of tile f - kSBufs had
            // completed, so pv_done of f - 1's buffer is at most one phase behind). Rows decide
            // separately; the O accesses are warp-collective, so the warp rescales its 64 columns
            // when any of its rows needs it (factor is 1 for the others).
            const long long fp = f - 1;
            wait(&sm.pv_done[ring_slot<kSBufs>(fp)], ring_phase<kSBufs>(fp), kDetailWaitPvDone);
            __syncwarp();
            tc_fence_after();
#pragma unroll 1
            for (int cb = 0; cb < 2; ++cb) {
              uint32_t orr[32];
              tmem_ld32(o_tm + 32u * (uint32_t)cb, orr);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * factor);
              tmem_st32(o_tm + 32u * (uint32_t)cb, orr);
            }
            tmem_wait_st();
          }
          if (h == 0 && k < gi.nctx && valid < kTile) {
            // Rows past the end of the context hold whatever the caller's slab or page holds
            // there; P is 0 for them, but 0 * NaN would still poison O, so zero those V rows
            // before the PV product reads them. The V tile must have landed first.
            const int stage = ring_slot<kVStages>(f);
            wait(&sm.v_full[stage], ring_phase<kVStages>(f), kDetailWaitKvFull);
            uint8_t* vbase = smem + kSmemV + stage * kKBytesPerStage;
            const int chunks_per_box = (kTile - valid) * 8;   // 16-byte chunks
            for (int i = t; i < 2 * chunks_per_box; i += kRows) {
              const int box = i / chunks_per_box, r = i - box * chunks_per_box;
              *reinterpret_cast<uint4*>(vbase + box * kKVBoxBytes + (valid + r / 8) * 128 + (r % 8) * 16) =
                  make_uint4(0u, 0u, 0u, 0u);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          }
          m_used = m_new;
          // every lane's TMEM stores (and O rescale) are complete and fenced before the warp's one
          // arrival hands P to the MMA thread
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.p_full[b]);
        }
        if (!ok) break;
        // ---- epilogue of the segment: wait for the last PV product, then the row's sum over both
        // halves, then this half's 64 dims of O / l
        wait(&sm.o_full, (uint32_t)(nseg & 1), kDetailWaitPvDone);
        float l_other;
        if (!exchange(l, l_other)) {
          ok = false;
          break;
        }
        const float l_all = l + l_other;
        __syncwarp();
        tc_fence_after();
        ++nseg;
        const bool whole = (kb == 0) && (ke == gi.ntiles);
        const bool row_valid = t < nrows;
        const int s_idx = qt * p.s_per_tile + t / p.G;
        const int hq = gi.kvh * p.G + t % p.G;
        const float inv_l = 1.0f / l_all;
        const float lse2 = m_used + log2f(l_all);
        // partial slot unique per (group, team, query tile)
        const size_t slot = ((size_t)w.u + (size_t)team) * (size_t)p.nq + (size_t)qt;
        __nv_bfloat16* orow = p.out + (((size_t)gi.b * p.S + s_idx) * p.Hq + hq) * kD + 64 * h;
        float* prow = partials + (slot * kRows + t) * kD + 64 * h;
#pragma unroll 1
        for (int cb = 0; cb < 2; ++cb) {
          uint32_t orr[32];
          tmem_ld32(o_tm + 32u * (uint32_t)cb, orr);
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
        if (row_valid && h == 0) {
          if (whole) {
            if (p.lse) p.lse[((size_t)gi.b * p.Hq + hq) * p.S + s_idx] = lse2 * 0.69314718055994531f;
          } else {
            plse[slot * kRows + t] = lse2;
          }
        }
        w.advance(p, hdr);
      }
    }
  }

  // ---- 3. teardown: all tensor-core work issued by the two MMA threads completes before TMEM
  // is released (on the normal path it already has; on an abort path this drains it)
  if ((warp == 1 || warp == 3) && lane == 0) {
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

}  // namespace one

// Merges the partials of groups cut between teams (flash-decoding combine):
//   O = sum_j 2^(lse_j - M) O_j / sum_j 2^(lse_j - M),  M = max_j lse_j.
// A CTA takes 32 query rows of one (group, query tile), 8 threads per row, each thread 16 of the
// 128 dims: for 4 contributors at a time it loads their log2-sum-exps (the 8 threads of a row read
// the same words) and its 64-byte slices of their rows together, and combines them against a
// running maximum (a moving base rescales what was accumulated: exact, the same up to rounding as
// the two-pass form). CTAs of a group that one team held whole return after reading the group's
// contributor range.
constexpr int kMergeRowsPerCta = 32;
constexpr int kMergeThreads = 256;   // 8 threads per row

struct MergeParams {
  int32_t S, Hq, Hkv, G, nq, s_per_tile, groups;
  __nv_bfloat16* out;
  float* lse;
  const uint8_t* ws;
  size_t off_meta, off_crange, off_partials, off_lse;
  const int32_t* skip_if;
};

__global__ void __launch_bounds__(kMergeThreads) attn_merge_kernel(const MergeParams p) {
  pdl_wait();
  if (skip_requested(p.skip_if)) return;
  const int u = blockIdx.x;             // group
  const int qt = blockIdx.z;            // query tile
  const int row = blockIdx.y * kMergeRowsPerCta + (threadIdx.x >> 3);
  const int part = threadIdx.x & 7;     // dims [16 part, 16 part + 16)
  const AttnMeta* meta = reinterpret_cast<const AttnMeta*>(p.ws + p.off_meta);
  // the two reads are independent: issued together, one round trip
  const long long T = meta->total_tiles;
  const int2 cr = reinterpret_cast<const int2*>(p.ws + p.off_crange)[u];   // teams holding group u
  if (T <= 0) return;
  const long long c_lo = cr.x, c_hi = cr.y;
  if (c_lo == c_hi) return;   // a whole group: the attention kernel wrote it
  const int kvh = u % p.Hkv, b = u / p.Hkv;
  const int s_cnt = min(p.s_per_tile, p.S - qt * p.s_per_tile);
  if (row >= p.G * s_cnt) return;
  const float* partials = reinterpret_cast<const float*>(p.ws + p.off_partials);
  const float* plse = reinterpret_cast<const float*>(p.ws + p.off_lse);
  const int n = (int)(c_hi - c_lo + 1);
  auto slot_of = [&](int j) { return ((size_t)u + (size_t)(c_lo + j)) * (size_t)p.nq + (size_t)qt; };
  // contributors 4 at a time, each batch's log2-sum-exps and 64-byte slices loaded together (one
  // round trip per batch); the running base moves with the batch maximum (online combine)
  float4 acc[4] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f),
                   make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
  float mx = -INFINITY, wsum = 0.f;
  for (int j0 = 0; j0 < n; j0 += 4) {
    float4 v[4][4];
    float wl[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      wl[q] = -INFINITY;
      if (j0 + q < n) {
        const size_t sl = slot_of(j0 + q);
        wl[q] = __ldg(plse + sl * kRows + row);
        const float4* src = reinterpret_cast<const float4*>(partials + (sl * kRows + row) * kD) + 4 * part;
#pragma unroll
        for (int c = 0; c < 4; ++c) v[q][c] = __ldg(src + c);
      }
    }
    const float bm = fmaxf(fmaxf(wl[0], wl[1]), fmaxf(wl[2], wl[3]));
    if (bm > mx) {
      // a new base: what was accumulated so far is scaled to it (factor 0 on the first batch)
      const float f = ex2(mx - bm);
      wsum *= f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        acc[c].x *= f;
        acc[c].y *= f;
        acc[c].z *= f;
        acc[c].w *= f;
      }
      mx = bm;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (j0 + q < n) {
        const float wq = ex2(wl[q] - mx);
        wsum += wq;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          acc[c].x = fmaf(wq, v[q][c].x, acc[c].x);
          acc[c].y = fmaf(wq, v[q][c].y, acc[c].y);
          acc[c].z = fmaf(wq, v[q][c].z, acc[c].z);
          acc[c].w = fmaf(wq, v[q][c].w, acc[c].w);
        }
      }
    }
  }
  const float inv = 1.0f / wsum;
  const int s_idx = qt * p.s_per_tile + row / p.G;
  const int hq = kvh * p.G + row % p.G;
  __nv_bfloat16* orow = p.out + (((size_t)b * p.S + s_idx) * p.Hq + hq) * kD + 16 * part;
  uint4 o0, o1;
  o0.x = pack_bf16x2(acc[0].x * inv, acc[0].y * inv);
  o0.y = pack_bf16x2(acc[0].z * inv, acc[0].w * inv);
  o0.z = pack_bf16x2(acc[1].x * inv, acc[1].y * inv);
  o0.w = pack_bf16x2(acc[1].z * inv, acc[1].w * inv);
  o1.x = pack_bf16x2(acc[2].x * inv, acc[2].y * inv);
  o1.y = pack_bf16x2(acc[2].z * inv, acc[2].w * inv);
  o1.z = pack_bf16x2(acc[3].x * inv, acc[3].y * inv);
  o1.w = pack_bf16x2(acc[3].z * inv, acc[3].w * inv);
  reinterpret_cast<uint4*>(orow)[0] = o0;
  reinterpret_cast<uint4*>(orow)[1] = o1;
  if (p.lse && part == 0) p.lse[((size_t)b * p.Hq + hq) * p.S + s_idx] = (mx + log2f(wsum)) * 0.69314718055994531f;
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

}  // namespace

bool attn_tc_supported(const tt_attn_args_t* a) {
  if (a->dtype != TT_BF16 || a->head_dim != kD) return false;
  const int G = a->num_q_heads / a->num_kv_heads;
  if (G > kRows) return false;                       // one block position's heads fit one query tile
  if (a->block_size > kTile) return false;
  if (a->page_table && (a->page_size % kTile) != 0) return false;   // a tile never crosses a page
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
  pl.s_per_tile = std::min(S, kRows / G);
  pl.qtiles = (S + pl.s_per_tile - 1) / pl.s_per_tile;        // nq
  pl.units = a->batch * a->num_kv_heads;                        // groups
  const int sms = std::max(1, num_sms);
  // Groups of one query tile run the one-tile kernel. Groups of two do too (a team of two CTAs,
  // one query tile each) when the CTAs would see few key tiles each: that kernel fills its
  // pipeline sooner and a group is cut among fewer teams, so the merge has fewer partials. The
  // lengths are on the device; the bound on the key tiles comes from the context capacity.
  const long long cap = a->page_table ? (long long)a->max_pages_per_seq * a->page_size : (long long)a->ctx_stride;
  const long long tiles_ub = (long long)pl.units * ((cap + kTile - 1) / kTile + 1);
  pl.one_tile = (pl.qtiles == 1 || (pl.qtiles == 2 && tiles_ub <= kOneTileMaxTilesPerSm * (long long)sms)) ? 1 : 0;
  pl.team_size = pl.one_tile ? pl.qtiles : (pl.qtiles + 1) / 2;   // CTAs per team
  const int teams = std::max(1, sms / pl.team_size);
  pl.grid = teams * pl.team_size;
  pl.slots = ((size_t)pl.units + (size_t)teams) * (size_t)pl.qtiles;
  size_t off = kHeaderBytes;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = (off + bytes + 255) & ~size_t(255);
    return o;
  };
  pl.off_meta = take(sizeof(AttnMeta));
  pl.off_crange = take(sizeof(int32_t) * 2 * (size_t)pl.units);
  pl.off_partials = take(sizeof(float) * pl.slots * kRows * kD);
  pl.off_lse = take(sizeof(float) * pl.slots * kRows);
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
  p.nq = pl.qtiles;
  p.nq2 = pl.team_size;
  p.s_per_tile = pl.s_per_tile;
  p.groups = pl.units;
  p.teams = pl.grid / pl.team_size;
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
  p.off_crange = pl.off_crange;
  p.off_partials = pl.off_partials;
  p.off_lse = pl.off_lse;
  p.skip_if = a->skip_if;
  // the shared-memory opt-ins are per device; set them once so no attribute call happens while a
  // caller captures the stream into a CUDA graph
  static unsigned long long attr_done = 0;   // bit per device ordinal (< 64)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TT_ERR_CUDA;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(__atomic_load_n(&attr_done, __ATOMIC_ACQUIRE) & bit)) {
    // The register raise of the softmax warpgroups waits until the block's pool (launch registers
    // x threads) has room: refuse to launch unless the compiled kernels start with enough.
    cudaFuncAttributes fa{}, fa1{};
    if (cudaFuncGetAttributes(&fa, attn_tc_kernel) != cudaSuccess ||
        cudaFuncGetAttributes(&fa1, one::attn_tc1_kernel) != cudaSuccess)
      return TT_ERR_CUDA;
    if (fa.numRegs * kThreads < 128 * kProducerRegs + 2 * 128 * kSoftmaxRegs) return TT_ERR_UNSUPPORTED;
    if (fa1.numRegs * one::kThreads < 128 * one::kProducerRegs + 2 * 128 * one::kSoftmaxRegs)
      return TT_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) !=
            cudaSuccess ||
        cudaFuncSetAttribute(one::attn_tc1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)one::kSmemBytes) != cudaSuccess)
      return TT_ERR_CUDA;
    __atomic_fetch_or(&attr_done, bit, __ATOMIC_ACQ_REL);
  }
  // the plan's choice: the one-tile kernel (both softmax warpgroups on one query tile per CTA) or
  // the two-stream kernel (two query tiles per CTA)
  const cudaError_t le =
      pl.one_tile
          ? launch_pdl(one::attn_tc1_kernel, dim3(pl.grid), dim3(one::kThreads), one::kSmemBytes, stream, p)
          : launch_pdl(attn_tc_kernel, dim3(pl.grid), dim3(kThreads), kSmemBytes, stream, p);
  if (le != cudaSuccess) return TT_ERR_CUDA;
  MergeParams mp{};
  mp.S = p.S;
  mp.Hq = p.Hq;
  mp.Hkv = p.Hkv;
  mp.G = G;
  mp.nq = pl.qtiles;
  mp.s_per_tile = pl.s_per_tile;
  mp.groups = pl.units;
  mp.out = p.out;
  mp.lse = p.lse;
  mp.ws = p.ws;
  mp.off_meta = pl.off_meta;
  mp.off_crange = pl.off_crange;
  mp.off_partials = pl.off_partials;
  mp.off_lse = pl.off_lse;
  mp.skip_if = a->skip_if;
  const int M = G * pl.s_per_tile;
  const dim3 mgrid(pl.units, (M + kMergeRowsPerCta - 1) / kMergeRowsPerCta, pl.qtiles);
  if (launch_pdl(attn_merge_kernel, mgrid, dim3(kMergeThreads), 0, stream, mp) != cudaSuccess) return TT_ERR_CUDA;
  return TT_OK;
}

}  // namespace tt
