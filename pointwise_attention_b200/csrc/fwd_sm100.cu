// fwd_sm100.cu -- bf16 forward of HSTU causal pointwise aggregated attention
// on sm_100a: TMA-staged Q/K/V tiles, tcgen05 MMAs with TMEM accumulators, a
// register epilogue for bias + SiLU + causal mask between the two MMAs, and
// the LayerNorm-over-heads + SiLU(U) gate in the same kernel.
//
// Operation: "HSTU (Generative Recommender)" model card, Exported PyTorch,
// HSTUBlock.forward (silu(q k^T)/t, tril, attn @ v, gate by silu(u));
// relative position / time bias: "HSTU Hierarchical Sequential Transduction
// Units", §1 and §3; post-pooling normalisation then U gate: the HSTU
// reproduction note's flowchart.
//
// Work decomposition.  A work item is one (sequence b, query tile m, head h):
// 128 query rows of one head against key tiles n = 0..m (tiles above the
// diagonal are skipped; only the diagonal tile is masked).  The kernel is
// persistent, one CTA per SM, and each CTA claims items from a counter in the
// workspace (its first item, slot c for CTA c, without a claim).  Slots are
// numbered heaviest first (largest m), the heads of one (b, m) next to each
// other, in groups of sequences whose K and V fit in L2 together.
//
// LayerNorm over heads.  The normalisation of a row needs all H heads of the
// row, which different CTAs compute at different times.  When a CTA finishes
// its head of a (b, m) block it stores O (bf16, less its per-row head mean,
// into the rows of Y that will later hold the result; fp32 into o_save when
// the caller keeps O) and the per-row statistics of its 128 values (mean, sum
// of squared deviations) in the workspace, then counts itself done on the
// block's counter.  The CTA that completes the count normalises and gates the
// whole 128 x (H*128) block: no CTA ever waits for another.
//
// Roles (608 threads): warp 0 claims items and issues TMA; warp 1 allocates
// TMEM and issues S = Q K^T; warp 2 issues O += P V (a tcgen05.mma of
// 128x128x16 occupies its issuing thread about as long as the tensor core
// needs for it, so the two GEMMs of a tile get one issuer each); warps 3..18
// are the epilogue: warp w owns TMEM lane quarter w%4 (rows 32*(w%4) ..) and
// the 32 columns (w-3)/4 of every tile, so all sixteen share each tile and
// its latency stays short against the three-buffer S -> P -> P.V cycle.  Each
// warp stages the position-bias diagonals and key timestamps of its own 32x32
// block in a private buffer, fetched from global memory one tile ahead.
//
// TMEM (512 columns): S/P buffers [0,128) [128,256) [256,384) and O
// [384,512).  P' = SiLU(S + bias) is written over S as packed bf16 pairs
// (keys 32c..32c+31 of column group c into columns 32c..32c+15, which that
// group's warps have already read) and is the A operand of O' += P' V;
// O = O' / N in the epilogue.  The bias add and SiLU
// run on bf16 pairs: hx = S/2 + bias/2, P' = hx (1 + tanh hx) with one
// tanh.approx.bf16x2 per two elements.
//
// Every tcgen05.ld/st is warp-collective (.sync.aligned) and issued with
// warp-uniform control flow; only global accesses are predicated per row.
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>

#include "bounds.cuh"
#include "internal.h"
#include "ptx.cuh"
#include "tile_math.cuh"

namespace hstu {
namespace {

constexpr int kRows = 128;                  // query rows per tile
constexpr int kCols = 128;                  // keys per tile
constexpr int kHalf = 16384;                // 128 rows x 64 bf16 (one 128B-swizzle slab)
constexpr int kTile = 2 * kHalf;            // 128 x 128 bf16
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr int kSBufs = 3;                   // S/P buffers in TMEM
constexpr int kRing = 8;                    // claimed items in flight inside the CTA
constexpr int kMaxHeads = 8;
constexpr int kWarpS = 1, kWarpPV = 2, kWarpEpi = 3;
constexpr int kEpiWarps = 16;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = (kWarpEpi + kEpiWarps) * 32;   // 608

// shared-memory map (byte offsets from a 1024-aligned base)
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kTile;
constexpr int kOffV = kOffK + kKStages * kTile;
// Per epilogue warp: the half position bias of the 63 diagonals its 32x32
// block touches, as 64 overlapping bf16 pairs (entry k holds diagonals k and
// k-1, the two an element pair needs); its 32 key timestamps (64-bit and low
// 32 bits).
constexpr int kWarpStage = 64 * 4 + 32 * 8 + 32 * 4;
constexpr int kOffWarp = kOffV + kVStages * kTile;
constexpr int kOffLoc = kOffWarp + kEpiWarps * kWarpStage;   // [4][128] (sum, M2) of O
constexpr int kOffRabT = kOffLoc + 4 * 128 * 8;              // 128 fp32 half time bias (item's head)
constexpr int kOffOct = kOffRabT + 128 * 4;
constexpr int kOffThr32 = kOffOct + 32 * 16;
constexpr int kOffThr = kOffThr32 + kMaxBuckets * 4;
constexpr int kOffFirst = kOffThr + kThrLen * 8;
constexpr int kOffRing = kOffFirst + 64;                     // kRing int4 {m, b, h, -}
constexpr int kOffBar = kOffRing + kRing * 16;
constexpr int kNumBars = 40;
constexpr int kOffMisc = kOffBar + kNumBars * 8;             // tmem base, abort flag, broadcast
constexpr int kSmemBytes = kOffMisc + 64 + 1024;             // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

// barrier indices
constexpr int B_QFULL = 0;
constexpr int B_QEMPTY = 1;
constexpr int B_KFULL = 2;    // +K stage
constexpr int B_KEMPTY = 5;   // +K stage
constexpr int B_VFULL = 8;    // +V stage
constexpr int B_VEMPTY = 10;  // +V stage
constexpr int B_SFULL = 12;   // +buffer: S(x) computed
constexpr int B_PFULL = 15;   // +buffer: P(x) written over S(x) (one arrival per epilogue warp)
constexpr int B_PVDONE = 18;  // +buffer: P(x).V completed, the buffer may be rewritten
constexpr int B_OFULL = 21;   // every P.V of the item completed
constexpr int B_OFREE = 22;   // O read out of TMEM (one arrival per epilogue warp)
constexpr int B_DONE = 23;    // every MMA of both issuers has completed
constexpr int B_RFULL = 24;   // +ring slot: item written
constexpr int B_REMPTY = 32;  // +ring slot: every role has read the item
static_assert(B_REMPTY + kRing == kNumBars, "barrier count");
constexpr uint32_t kRingReaders = 2 + kEpiWarps;   // both issuers + each epilogue warp
constexpr int kTmemCols = 512;
constexpr uint32_t kColO = 384;
// named barriers of the epilogue warps (0 is __syncthreads)
constexpr int NB_EXIT = 1;    // OR-reduced decisions to stop
constexpr int NB_SYNC = 2;

constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false, false);   // Q (K-major) x K (K-major)
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, false, true);   // P (TMEM) x V (MN-major)

__device__ __forceinline__ void set_status(int* status, int bit) {
  if (status) atomicOr(status, bit);
}

// Passes a bounded wait's result through; when it failed, records the
// timeout bit and, for the first failure of the launch, where it happened in
// status words 2..5 (wait site, CTA, item, tile) for diagnosis.
__device__ __forceinline__ bool waited(bool r, int* status, int site, int j, int x) {
  if (!r && status) {
    atomicOr(status, kStatusTimeout);
    if (atomicCAS(status + 2, 0, site) == 0) {
      status[3] = static_cast<int>(blockIdx.x);
      status[4] = j;
      status[5] = x;
    }
  }
  return r;
}

// SiLU of a pair of half arguments hx = x/2: x/2 (1 + tanh(x/2)) = SiLU(x).
__device__ __forceinline__ uint32_t silu_pair(uint32_t hx) { return hfma2(hx, tanh2(hx), hx); }

// SiLU of the gate input through tanh: x/2 (1 + tanh(x/2)).
__device__ __forceinline__ float silu_gate(float x) {
  const float hx = 0.5f * x;
  return fmaf(hx, tanh_approx(hx), hx);
}

// Start and length of sequence b; inconsistent offsets give length -1.
__device__ __forceinline__ int2 load_seq(const FwdArgs& a, int b, bool pos) {
  const int s = __ldg(a.offsets + b);
  const int e = __ldg(a.offsets + b + 1);
  const int n = e - s;
  if (s < 0 || n < 0 || e > a.T || n > a.max_seq_len || (pos && n > a.L)) return make_int2(0, -1);
  return make_int2(s, n);
}

// Work slots: sequences are taken in groups of G whose keys and values fit in
// L2 together; inside a group, slot r is the item (m = M-1 - r/(G H),
// b = group * G + (r / H) mod G, h = r mod H): the most expensive query tiles
// of the group come first (a longest-first list schedule) and the heads of
// one (b, m) block are claimed together.
struct Item {
  int m, b, h;
};

__device__ __forceinline__ Item slot_item(unsigned k, unsigned G, int M, int H) {
  const unsigned GH = G * static_cast<unsigned>(H);
  const unsigned per = GH * static_cast<unsigned>(M);
  const unsigned grp = k / per, r = k % per;
  const unsigned rest = r % GH;
  return Item{M - 1 - static_cast<int>(r / GH), static_cast<int>(grp * G + rest / H),
              static_cast<int>(rest % static_cast<unsigned>(H))};
}

// Claims the CTA's next item (warp-collective).  The CTA's first item is slot
// `first` (its block index) without touching the counter; every later claim
// takes slot base + the counter's old value from an atomic add.  A slot whose
// tile lies past its sequence end holds no work: the warp then tests the 31
// slots after it and raises the counter past the empty ones among them
// (atomicMax; every skipped slot was seen empty, and no slot is handed out
// twice), then claims again.  Returns m = -1 once the slots are exhausted.
template <bool POS>
__device__ Item claim_item(const FwdArgs& a, unsigned* counter, unsigned nslots, unsigned base,
                           int first, int lane) {
  const unsigned G = static_cast<unsigned>(a.group);
  const int M = a.max_tiles;
  bool fixed = first >= 0;
  for (;;) {
    unsigned k = static_cast<unsigned>(first);
    if (!fixed) {
      if (lane == 0) k = atomicAdd(counter, 1u) + base;
      k = __shfl_sync(0xffffffffu, k, 0);
    }
    if (k >= nslots) return Item{-1, -1, -1};
    const unsigned slot = k + static_cast<unsigned>(lane);
    bool valid = false;
    if (slot < nslots && (!fixed || lane == 0)) {
      const Item it = slot_item(slot, G, M, a.H);
      if (it.b < a.B) {   // the last group may be partial
        const int2 sq = load_seq(a, it.b, POS);
        if (sq.y < 0) {
          if (it.m == 0 && it.h == 0) set_status(a.status, kStatusBadOffsets);
        } else {
          valid = kRows * it.m < sq.y;
        }
      }
    }
    const unsigned vb = __ballot_sync(0xffffffffu, valid);
    if (vb & 1u) return slot_item(k, G, M, a.H);
    if (fixed) {          // the CTA's own first slot is empty: claim from the counter
      fixed = false;
      continue;
    }
    const unsigned rest = vb & ~1u;
    const unsigned skip_to = rest ? k + static_cast<unsigned>(__ffs(rest) - 1) : k + 32u;
    if (lane == 0 && skip_to > k + 1) atomicMax(counter, min(skip_to, nslots) - base);
  }
}

// Time bias of one 32-key chunk for one row, as the element loop takes it:
// one value (CONST) or two with a split column (SPLIT), from the row's plan
// word (plans.cu); every other plan kind takes each element's own bucket
// (GEN32 with 32-bit differences, GEN64 for time spans of 2^31 or more).
enum { T_CONST = 0, T_SPLIT = 1, T_GEN32 = 2, T_GEN64 = 3, T_MULTI = 4, T_BYTES = 5 };

struct EpiShared {
  const uint4* oct;
  const unsigned* thr32;
  const long long* thr;
  const signed char* first;
  const float* rabt;         // half time bias per bucket
};

// P' pairs of one 32-column chunk: sv = S (fp32), wpk = the warp's staged
// position-bias pairs, indexed (lane - 2i + 31) for columns 2i, 2i+1 (halved
// bf16), result packed[16].  TM selects the time plan.
template <bool POS, bool TIME, int TM>
__device__ __forceinline__ void chunk_pairs(const uint32_t (&sv)[32], const uint32_t* wpk,
                                            uint32_t tconst, uint32_t thh, uint32_t tll,
                                            uint32_t thl, int split, uint32_t my32,
                                            long long my64, const uint32_t* kts32,
                                            const long long* kts64, const EpiShared& es,
                                            uint32_t (&packed)[16], const uint32_t* nbw = nullptr) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t s2 = pack_bf16x2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1]));
    uint32_t hx = hfma2(s2, kHalfPair, POS ? wpk[-2 * i] : 0u);
    if (TIME) {
      uint32_t tb;
      if (TM == T_CONST) {
        tb = tconst;
      } else if (TM == T_SPLIT) {
        tb = (2 * i + 1 < split) ? thh : ((2 * i < split) ? thl : tll);
      } else if (TM == T_MULTI) {
        // splits in `split` (6 bits each), the four bucket values in
        // tconst, thh, tll, thl
        const int s0 = split & 63, s1 = (split >> 6) & 63, s2 = (split >> 12) & 63;
        const int c = 2 * i;
        const uint32_t lo = c >= s2 ? thl : c >= s1 ? tll : c >= s0 ? thh : tconst;
        const uint32_t hi = c + 1 >= s2 ? thl : c + 1 >= s1 ? tll : c + 1 >= s0 ? thh : tconst;
        tb = __byte_perm(lo, hi, 0x7610);
      } else if (TM == T_BYTES) {
        // each element's bucket from the plan pass, one byte per column
        const int2 kb = byte_bucket_pair(nbw, i);
        tb = pack_bf16x2(es.rabt[kb.x], es.rabt[kb.y]);
      } else {
        float tv[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          int k;
          if (TM == T_GEN32) {
            const int d = static_cast<int>(my32 - kts32[2 * i + hh]);
            k = bucket32(static_cast<uint32_t>(d < 0 ? -d : d), es.oct);
          } else {
            k = time_bucket(my64 - kts64[2 * i + hh], es.thr, es.first);
          }
          tv[hh] = es.rabt[k];
        }
        tb = pack_bf16x2(tv[0], tv[1]);
      }
      hx = hadd2(hx, tb);
    }
    packed[i] = silu_pair(hx);
  }
}

template <bool POS, bool TIME>
__global__ void __launch_bounds__(kThreads, 1)
    hstu_fwd_bf16_sm100(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ FwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int H = a.H;

  auto bar = [&](int i) { return sbase + kOffBar + 8u * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  int4* ring = reinterpret_cast<int4*>(smem + kOffRing);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      uint32_t count = 1;
      if ((i >= B_PFULL && i < B_PFULL + kSBufs) || i == B_OFREE) count = kEpiWarps;
      if (i == B_DONE) count = 2;                                        // both issuers
      if (i >= B_REMPTY && i < B_REMPTY + kRing) count = kRingReaders;
      mbar_init(bar(i), count);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpS) {
    tmem_alloc(sbase + kOffMisc, kTmemCols);
    tmem_relinquish();
  }
  if (TIME && warp >= kWarpEpi) {
    const int et = threadIdx.x - kWarpEpi * 32;
    long long* s_thr = reinterpret_cast<long long*>(smem + kOffThr);
    for (int i = et; i < kThrLen; i += kEpiThreads) s_thr[i] = a.bt.thr[i];
    if (et < kMaxBuckets) reinterpret_cast<unsigned*>(smem + kOffThr32)[et] = a.bt.thr32[et];
    if (et < 32) reinterpret_cast<uint4*>(smem + kOffOct)[et] = a.bt.oct[et];
    if (et < 64) reinterpret_cast<signed char*>(smem + kOffFirst)[et] = a.bt.first_k[et];
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  auto wait_item = [&](int j) -> bool {
    return waited(mbar_wait(bar(B_RFULL + j % kRing), (j / kRing) & 1, abort_flag), a.status,
                  warp < kWarpEpi ? 10 + warp : 20, j, -1);
  };
  auto read_item = [&](int j) -> Item {
    const int4 v = ring[j % kRing];
    return Item{v.x, v.y, v.z};
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    unsigned* counter = reinterpret_cast<unsigned*>(a.status) + kSchedCounterWord;
    unsigned* done = reinterpret_cast<unsigned*>(a.status) + kSchedDoneWord;
    const unsigned nslots = static_cast<unsigned>((a.B + a.group - 1) / a.group) *
                            static_cast<unsigned>(a.group) * static_cast<unsigned>(a.max_tiles) *
                            static_cast<unsigned>(H);
    // Claim item j and publish it in the ring (warp-collective).
    auto fetch = [&](int j) -> Item {
      bool okf = true;
      if (lane == 0 && j >= kRing)
        okf = waited(mbar_wait(bar(B_REMPTY + j % kRing), ((j / kRing) - 1) & 1, abort_flag),
                     a.status, 1, j, -1);
      okf = __shfl_sync(0xffffffffu, okf, 0);
      if (!okf) return Item{-2, -2, -2};
      const Item it = claim_item<POS>(a, counter, nslots, gridDim.x,
                                      j == 0 ? static_cast<int>(blockIdx.x) : -1, lane);
      if (lane == 0) {
        ring[j % kRing] = make_int4(it.m, it.b, it.h, 0);
        mbar_arrive(bar(B_RFULL + j % kRing));
      }
      __syncwarp();
      return it;
    };

    int k_last[kKStages] = {-1, -1, -1}, v_last[kVStages] = {-1, -1};
    int q_last = -1;
    bool ok = true;
    int j = 0, g = 0;
    Item it = fetch(0);
    while (it.m >= 0) {
      if (lane == 0) {
        const int m = it.m, nt = m + 1, h = it.h;
        const int s = __ldg(a.offsets + it.b);
        if (j > 0) ok = waited(mbar_wait(bar(B_QEMPTY), (j - 1) & 1, abort_flag), a.status, 2, j, g);
        if (ok) {
          const int row0 = checked(a.status, s + kRows * m, a.T, BS_FWD_TMA_Q);
          mbar_arrive_expect_tx(bar(B_QFULL), kTile);
          tma_load_3d(sbase + kOffQ, &tm_q, bar(B_QFULL), 0, h, row0);
          tma_load_3d(sbase + kOffQ + kHalf, &tm_q, bar(B_QFULL), 64, h, row0);
          q_last = j;
        }
        // K runs one tile ahead of V: K(x+1) is requested before V(x), whose
        // stage frees only when P(x-2).V completes.  x is the running tile index.
        auto load_k = [&](int x, int n) -> bool {
          const int st = x % kKStages, use = x / kKStages;
          if (use > 0 && !waited(mbar_wait(bar(B_KEMPTY + st), (use - 1) & 1, abort_flag), a.status,
                                 3, j, x))
            return false;
          const int krow = checked(a.status, s + kCols * n, a.T, BS_FWD_TMA_KV);
          mbar_arrive_expect_tx(bar(B_KFULL + st), kTile);
          tma_load_3d(sbase + kOffK + st * kTile, &tm_k, bar(B_KFULL + st), 0, h, krow);
          tma_load_3d(sbase + kOffK + st * kTile + kHalf, &tm_k, bar(B_KFULL + st), 64, h, krow);
          k_last[st] = use;
          return true;
        };
        auto load_v = [&](int x, int n) -> bool {
          const int st = x % kVStages, use = x / kVStages;
          if (use > 0 && !waited(mbar_wait(bar(B_VEMPTY + st), (use - 1) & 1, abort_flag), a.status,
                                 4, j, x))
            return false;
          const int krow = checked(a.status, s + kCols * n, a.T, BS_FWD_TMA_KV);
          mbar_arrive_expect_tx(bar(B_VFULL + st), kTile);
          tma_load_3d(sbase + kOffV + st * kTile, &tm_v, bar(B_VFULL + st), 0, h, krow);
          tma_load_3d(sbase + kOffV + st * kTile + kHalf, &tm_v, bar(B_VFULL + st), 64, h, krow);
          v_last[st] = use;
          return true;
        };
        if (ok) ok = load_k(g, 0);
        for (int n = 0; n < nt && ok; ++n) {
          if (n + 1 < nt) ok = load_k(g + n + 1, n + 1);
          if (ok) ok = load_v(g + n, n);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      g += it.m + 1;
      ++j;
      it = fetch(j);
    }
    if (it.m == -2) ok = false;
    if (!ok && lane == 0) {
      // Let the other roles leave: publish an end marker where they wait next.
      ring[j % kRing] = make_int4(-2, -2, -2, 0);
      mbar_arrive(bar(B_RFULL + j % kRing));
    }
    if (lane == 0) {
      if (!ok) {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
        // Let the copies already issued land before shared memory goes away.
        if (q_last >= 0) mbar_wait(bar(B_QFULL), q_last & 1, nullptr);
        for (int st = 0; st < kKStages; ++st)
          if (k_last[st] >= 0) mbar_wait(bar(B_KFULL + st), k_last[st] & 1, nullptr);
        for (int st = 0; st < kVStages; ++st)
          if (v_last[st] >= 0) mbar_wait(bar(B_VFULL + st), v_last[st] & 1, nullptr);
      }
      // The last CTA to finish returns the work counter to zero for the next launch.
      __threadfence();
      if (atomicAdd(done, 1u) == gridDim.x - 1) {
        atomicExch(counter, 0u);
        atomicExch(done, 0u);
      }
    }
  } else if (warp == kWarpS) {
    // ------------------------------------------------------------ S issuer
    if (lane == 0) {
      bool ok = true;
      int j = 0, g = 0;
      for (;;) {
        ok = wait_item(j);
        if (!ok) break;
        const Item it = read_item(j);
        mbar_arrive(bar(B_REMPTY + j % kRing));
        if (it.m < 0) break;
        const int nt = it.m + 1;
        ok = waited(mbar_wait(bar(B_QFULL), j & 1, abort_flag), a.status, 5, j, g);
        for (int n = 0; n < nt && ok; ++n) {
          const int x = g + n, st = x % kKStages, buf = x % kSBufs;
          // The buffer's previous tile x-3 has been consumed by its P.V.
          if (x >= kSBufs)
            ok = waited(mbar_wait(bar(B_PVDONE + buf), ((x - kSBufs) / kSBufs) & 1, abort_flag),
                        a.status, 6, j, x);
          if (ok)
            ok = waited(mbar_wait(bar(B_KFULL + st), (x / kKStages) & 1, abort_flag), a.status, 7, j,
                        x);
          if (!ok) break;
          tc_fence_after();
          const uint32_t d = tmem + 128u * buf;
          const uint32_t qa = sbase + kOffQ, ka = sbase + kOffK + st * kTile;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t off = (ks >> 2) * kHalf + (ks & 3) * 32;
            mma_ss(d, sw128_desc(qa + off, 16, 1024), sw128_desc(ka + off, 16, 1024), kIdescS,
                   ks > 0);
          }
          mma_commit(bar(B_KEMPTY + st));
          mma_commit(bar(B_SFULL + buf));
        }
        if (!ok) break;
        mma_commit(bar(B_QEMPTY));   // Q may be replaced by the next item's
        g += nt;
        ++j;
      }
      if (!ok) {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
      }
      mma_commit(bar(B_DONE));   // arrives once every MMA it issued has finished
    }
  } else if (warp == kWarpPV) {
    // ------------------------------------------------------------ P.V issuer
    if (lane == 0) {
      bool ok = true;
      int j = 0, g = 0;
      for (;;) {
        ok = wait_item(j);
        if (!ok) break;
        const Item it = read_item(j);
        mbar_arrive(bar(B_REMPTY + j % kRing));
        if (it.m < 0) break;
        const int nt = it.m + 1;
        // The previous item's O has been read out of TMEM.
        if (j > 0) ok = waited(mbar_wait(bar(B_OFREE), (j - 1) & 1, abort_flag), a.status, 8, j, g);
        for (int n = 0; n < nt && ok; ++n) {
          const int x = g + n, st = x % kVStages, buf = x % kSBufs;
          ok = waited(mbar_wait(bar(B_PFULL + buf), (x / kSBufs) & 1, abort_flag), a.status, 9, j, x);
          if (ok)
            ok = waited(mbar_wait(bar(B_VFULL + st), (x / kVStages) & 1, abort_flag), a.status, 30,
                        j, x);
          if (!ok) break;
          tc_fence_after();
          const uint32_t va = sbase + kOffV + st * kTile;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            // Keys 16ks..16ks+15: column group ks/2 holds its 32 keys in its
            // first 16 columns; rows 16ks.. of the V tile, whose two
            // 64-column halves of d_v are 16 KB apart (leading byte offset).
            mma_ts(tmem + kColO, tmem + 128u * buf + 32u * (ks >> 1) + 8u * (ks & 1),
                   sw128_desc(va + ks * 2048, kHalf, 1024), kIdescPV, (n > 0 || ks > 0));
          }
          mma_commit(bar(B_VEMPTY + st));
          mma_commit(bar(B_PVDONE + buf));
        }
        if (!ok) break;
        mma_commit(bar(B_OFULL));
        g += nt;
        ++j;
      }
      if (!ok) {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
      }
      mma_commit(bar(B_DONE));
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - kWarpEpi;               // 0..15
    const int q4 = warp & 3;                      // TMEM lane quarter
    const int cq = ew >> 2;                       // 32-column group of the S/P and O tiles
    const int r = q4 * 32 + lane;                 // row within the tile
    const int et = threadIdx.x - kWarpEpi * 32;   // 0..511 among epilogue threads
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    const int Lw = 2 * a.L - 1;
    const int D = H * 128;
    uint8_t* wstage = smem + kOffWarp + ew * kWarpStage;
    uint32_t* wpk = reinterpret_cast<uint32_t*>(wstage);
    long long* wts = reinterpret_cast<long long*>(wstage + 64 * 4);
    uint32_t* wts32 = reinterpret_cast<uint32_t*>(wstage + 64 * 4 + 32 * 8);
    float2* loc = reinterpret_cast<float2*>(smem + kOffLoc);   // [4][128]
    float* s_rabt = reinterpret_cast<float*>(smem + kOffRabT);
    volatile unsigned* bcast = reinterpret_cast<volatile unsigned*>(misc + 2);
    EpiShared es;
    es.oct = reinterpret_cast<const uint4*>(smem + kOffOct);
    es.thr32 = reinterpret_cast<const unsigned*>(smem + kOffThr32);
    es.thr = reinterpret_cast<const long long*>(smem + kOffThr);
    es.first = reinterpret_cast<const signed char*>(smem + kOffFirst);
    es.rabt = s_rabt;
    bool ok = true;
    int j = 0, g = 0;

    // Named barriers cannot time out, so every epilogue warp leaves the loop
    // at the same point: the decisions to stop are OR-reduced over all of them.
    for (;;) {
      const bool got = __all_sync(0xffffffffu, wait_item(j));
      const Item it = got ? read_item(j) : Item{-2, -2, -2};
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_REMPTY + j % kRing));
      // The previous item's last use of the time-bias row precedes the
      // barriers at its end: the row of this item's head replaces it here.
      if (TIME && got && it.m >= 0 && et < a.nb)
        s_rabt[et] = 0.5f * __ldg(a.rab_time + static_cast<size_t>(it.h) * a.nb + et);
      if (named_bar_or(NB_EXIT, kEpiThreads, !ok || it.m < 0)) {
        if (it.m == -2) ok = false;
        break;
      }
      const int m = it.m, nt = m + 1, b = it.b, h = it.h;
      const int s = __ldg(a.offsets + b);
      const int n_b = __ldg(a.offsets + b + 1) - s;
      const int i_loc = kRows * m + r;            // local row index in the sequence
      const bool row_ok = i_loc < n_b;
      const int t_row = s + (row_ok ? i_loc : 0);
      const float nrm = a.norm_len > 0 ? static_cast<float>(a.norm_len) : static_cast<float>(n_b);
      // Rows past the sequence end (never stored) take the last token's
      // timestamp: every key is then at or before them and the plans stay cheap.
      long long my64 = 0;
      if (TIME) my64 = a.timestamps[checked(a.status, row_ok ? t_row : s + n_b - 1, a.T, BS_FWD_TS)];
      const uint32_t my32 = static_cast<uint32_t>(my64);
      // The gate input of this row is read at the end of the block: ask L2 for it now.
      if (row_ok)
        prefetch_l2(reinterpret_cast<const __nv_bfloat16*>(a.u) + static_cast<size_t>(t_row) * D +
                    h * 128 + 32 * cq);

      // Staging of this warp's 32 x 32 block of tile n: half position bias of
      // the 63 diagonals d = r - c in [32 q4 - 32 cq - 31, 32 q4 - 32 cq + 31]
      // (table index 128 (m - n) + d + L - 1), entry k as the bf16 pair
      // (diagonal k, diagonal k-1), the timestamps of its 32 keys for the
      // per-element paths (keys past the sequence end repeat its last
      // timestamp; those keys are masked anyway) and this row's plan word.
      const int dbase = 32 * q4 - 32 * cq - 31;
      float pre_w0 = 0.f, pre_w1 = 0.f;
      long long pre_t = 0;
      uint32_t pre_w = 0, plan_w = 0;             // time plan word: prefetched, current
      auto prefetch = [&](int n) {
        if (POS) {
          const int t0 = kRows * (m - n) + dbase + lane + a.L - 1;
          const float* tab = a.rab_pos + static_cast<size_t>(h) * Lw;
          pre_w0 = (t0 >= 0 && t0 < Lw) ? __ldg(tab + t0) : 0.f;
          pre_w1 = (lane < 31 && t0 + 32 >= 0 && t0 + 32 < Lw) ? __ldg(tab + t0 + 32) : 0.f;
        }
        if (TIME) {
          const int jj = kCols * n + 32 * cq + lane;
          pre_t = a.timestamps[checked(a.status, s + (jj < n_b ? jj : n_b - 1), a.T, BS_FWD_TS)];
          // this row's time plan against the block (rows past the end read the last row's)
          pre_w = a.plan_dn[static_cast<size_t>(4 * n + cq) * a.T +
                            checked(a.status, row_ok ? t_row : s + n_b - 1, a.T, BS_FWD_TS)];
        }
      };
      auto stage = [&]() {   // this warp's previous reads of its buffer are done
        if (POS) {
          const float v0 = 0.5f * pre_w0, v1 = 0.5f * pre_w1;
          float p0 = __shfl_up_sync(0xffffffffu, v0, 1);
          float p1 = __shfl_up_sync(0xffffffffu, v1, 1);
          const float e0 = __shfl_sync(0xffffffffu, v0, 31);
          if (lane == 0) {
            p0 = 0.f;
            p1 = e0;
          }
          wpk[lane] = pack_bf16x2(v0, p0);        // low half: diagonal k
          wpk[32 + lane] = pack_bf16x2(v1, p1);
        }
        if (TIME) {
          wts[lane] = pre_t;
          wts32[lane] = static_cast<uint32_t>(pre_t);
          plan_w = pre_w;
        }
        __syncwarp();
      };

      prefetch(0);
      stage();
      for (int n = 0; n < nt; ++n) {
        const int x = g + n, buf = x % kSBufs;
        if (n + 1 < nt) prefetch(n + 1);          // global loads overlap this tile
        if (ok)
          ok = waited(mbar_wait(bar(B_SFULL + buf), (x / kSBufs) & 1, abort_flag), a.status, 40,
                      j, x);
        // The TMEM accesses below are warp-collective: keep the decision warp-uniform.
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;                           // on to the collective exit below
        tc_fence_after();
        const uint32_t s_addr = tmem + lane_addr + 128u * buf;
        uint32_t packed[16];
        const bool diag = (n == m);
        if (diag && cq > q4) {                    // entirely above the diagonal
#pragma unroll
          for (int i = 0; i < 16; ++i) packed[i] = 0u;
        } else {
          uint32_t sv[32];
          tmem_ld32_nowait(s_addr + 32u * cq, sv);
          tmem_wait_ld_dep(sv);
          // element (lane, c) uses diagonal index lane - c + 31
          const uint32_t* wp = wpk + 31 + lane;
          if (!TIME) {
            chunk_pairs<POS, false, T_CONST>(sv, wp, 0u, 0u, 0u, 0u, 0, 0u, 0ll, nullptr,
                                             nullptr, es, packed);
          } else {
            // this row's plan against the block's 32 keys (the time-plan pass):
            // the first key's bucket k0, the first column of bucket k0 - 1
            const int kind = static_cast<int>(plan_w >> 25) & 7;
            const int k0 = static_cast<int>(plan_w & 127u);
            if (kind == TB_CONST) {
              const float tv = es.rabt[k0];
              chunk_pairs<POS, true, T_CONST>(sv, wp, pack_bf16x2(tv, tv), 0u, 0u, 0u, 0, my32,
                                              my64, wts32, wts, es, packed);
            } else if (kind == TB_SPLIT) {
              const int split = static_cast<int>((plan_w >> 7) & 63u);
              const float hv = es.rabt[k0], lv = es.rabt[k0 > 0 ? k0 - 1 : 0];
              chunk_pairs<POS, true, T_SPLIT>(sv, wp, 0u, pack_bf16x2(hv, hv),
                                              pack_bf16x2(lv, lv), pack_bf16x2(hv, lv), split,
                                              my32, my64, wts32, wts, es, packed);
            } else if (kind == TB_MULTI) {
              // the word's three split columns and the buckets k0 .. k0 - 3
              const float v0 = es.rabt[k0], v1 = es.rabt[max(k0 - 1, 0)];
              const float v2 = es.rabt[max(k0 - 2, 0)], v3 = es.rabt[max(k0 - 3, 0)];
              chunk_pairs<POS, true, T_MULTI>(sv, wp, pack_bf16x2(v0, v0), pack_bf16x2(v1, v1),
                                              pack_bf16x2(v2, v2), pack_bf16x2(v3, v3),
                                              static_cast<int>((plan_w >> 7) & 0x3FFFFu), my32,
                                              my64, wts32, wts, es, packed);
            } else if (kind != TB_GEN64) {               // per element
              const int jd = 4 * m + q4, jc = 4 * n + cq;   // diagonal block, this block
              if (jc == jd || jc == jd - 1) {
                // the buckets of the two blocks nearest the diagonal, from the plan pass
                const uint4* src = a.near +
                                   static_cast<size_t>(row_ok ? t_row : s + n_b - 1) * 6 +
                                   (jc == jd ? 0 : 2);
                const uint4 b0 = __ldg(src), b1 = __ldg(src + 1);
                const uint32_t nbw[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                chunk_pairs<POS, true, T_BYTES>(sv, wp, 0u, 0u, 0u, 0u, 0, my32, my64, wts32, wts,
                                                es, packed, nbw);
              } else {
                chunk_pairs<POS, true, T_GEN32>(sv, wp, 0u, 0u, 0u, 0u, 0, my32, my64, wts32,
                                                wts, es, packed);
              }
            } else {
              chunk_pairs<POS, true, T_GEN64>(sv, wp, 0u, 0u, 0u, 0u, 0, my32, my64, wts32, wts,
                                              es, packed);
            }
          }
          if (diag && cq == q4) {                 // causal mask: column 32 cq + c > row r
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const uint32_t keep = (2 * i > lane ? 0u : 0x0000FFFFu) |
                                    (2 * i + 1 > lane ? 0u : 0xFFFF0000u);
              packed[i] &= keep;
            }
          }
        }
        tmem_st16(s_addr + 32u * cq, packed);   // over this warp's own, already read S columns
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_PFULL + buf));
        if (n + 1 < nt) stage();
      }

      // -------------------------------------- O of the item: statistics and stash
      if (named_bar_or(NB_EXIT, kEpiThreads, !ok)) {
        ok = false;
        break;
      }
      ok = waited(mbar_wait(bar(B_OFULL), j & 1, abort_flag), a.status, 50, j, g + nt - 1);
      ok = __all_sync(0xffffffffu, ok);
      float ov[32];
      {
        uint32_t o0[32];
        if (ok) {
          tc_fence_after();
          tmem_ld32_nowait(tmem + lane_addr + kColO + 32u * cq, o0);
          tmem_wait_ld_dep(o0);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o0[i] = 0u;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_OFREE));   // the next item's P.V may overwrite O
        const float inv_n = 1.0f / nrm;             // O accumulated SiLU(.) terms
#pragma unroll
        for (int i = 0; i < 32; ++i) ov[i] = __uint_as_float(o0[i]) * inv_n;
      }
      {
        // sum and sum of squared deviations of this thread's 32 values
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) sum += ov[i];
        const float mu = sum * (1.0f / 32.0f);
        float m2 = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float d0 = ov[i] - mu;
          m2 = fmaf(d0, d0, m2);
        }
        loc[cq * 128 + r] = make_float2(sum, m2);
      }
      named_bar_sync(NB_SYNC, kEpiThreads);
      // The head's (mean, M2) of the row from its four 32-column groups.
      const float2 p0 = loc[r], p1 = loc[128 + r], p2 = loc[256 + r], p3 = loc[384 + r];
      const float mean_h = ((p0.x + p1.x) + (p2.x + p3.x)) * (1.0f / 128.0f);
      const float e0 = p0.x * (1.0f / 32.0f) - mean_h, e1 = p1.x * (1.0f / 32.0f) - mean_h;
      const float e2 = p2.x * (1.0f / 32.0f) - mean_h, e3 = p3.x * (1.0f / 32.0f) - mean_h;
      const float m2_h = (p0.y + p1.y) + (p2.y + p3.y) +
                         32.0f * ((e0 * e0 + e1 * e1) + (e2 * e2 + e3 * e3));
      const size_t rowD = static_cast<size_t>(t_row) * D + static_cast<size_t>(h) * 128 + 32 * cq;
      if (ok && row_ok) {
        if (a.o_save) {
          float* od = a.o_save + rowD;
          if (a.vec32) {
#pragma unroll
            for (int v = 0; v < 4; ++v)
              st_global_v8(od + 8 * v, reinterpret_cast<const uint32_t(&)[8]>(ov[8 * v]));
          } else {
#pragma unroll
            for (int v = 0; v < 8; ++v)
              reinterpret_cast<float4*>(od)[v] =
                  make_float4(ov[4 * v], ov[4 * v + 1], ov[4 * v + 2], ov[4 * v + 3]);
          }
        } else {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(ov[2 * i] - mean_h, ov[2 * i + 1] - mean_h);
          __nv_bfloat16* yd = reinterpret_cast<__nv_bfloat16*>(a.y) + rowD;
          if (a.vec32) {
            st_global_v8(yd, reinterpret_cast<const uint32_t(&)[8]>(w[0]));
            st_global_v8(yd + 16, reinterpret_cast<const uint32_t(&)[8]>(w[8]));
          } else {
#pragma unroll
            for (int v = 0; v < 4; ++v)
              reinterpret_cast<uint4*>(yd)[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2],
                                                           w[4 * v + 3]);
          }
        }
        if (cq == 0)
          a.stats[static_cast<size_t>(t_row) * H + h] =
              make_float4(mean_h, m2_h, a.o_save ? 0.f : mean_h, 0.f);
      }
      // ---- count this head done on the (b, m) block; the last one normalises it.
      // Release: each thread fences its stash and statistics stores before
      // the barrier, then one thread counts; acquire: that thread fences
      // after the count, and every thread again after the barrier, before
      // reading the other heads' data.
      __threadfence();
      named_bar_sync(NB_SYNC, kEpiThreads);      // also: every loc read is done
      if (et == 0) {
        __threadfence();
        const unsigned old = atomicAdd(a.item_cnt + static_cast<size_t>(b) * a.max_tiles + m, 1u);
        __threadfence();
        *bcast = old;
      }
      named_bar_sync(NB_SYNC, kEpiThreads);
      if (ok && *bcast == static_cast<unsigned>(H - 1)) {
        __threadfence();
        // ---------------------------------- LayerNorm over heads + gate, rows of the block
        const int nrows = min(kRows, n_b - kRows * m);
        const bool fp32_stash = a.o_save != nullptr;
        const float invD = 1.0f / static_cast<float>(D);
        for (int rr = ew; rr < nrows; rr += kEpiWarps) {
          const int t = checked(a.status, s + kRows * m + rr, a.T, BS_FWD_ROW);
          float4 st = make_float4(0.f, 0.f, 0.f, 0.f);
          if (lane < H) st = ld_global_cg_f4(a.stats + static_cast<size_t>(t) * H + lane);
          float tot = lane < H ? st.x : 0.f;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
          const float mean = tot / static_cast<float>(H);
          const float dh = st.x - mean;
          float m2 = lane < H ? st.y + 128.0f * dh * dh : 0.f;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) m2 += __shfl_xor_sync(0xffffffffu, m2, o);
          const float rstd = 1.0f / sqrtf(m2 * invD + a.eps);
          // value = stash + shift_h, with shift_h = mean_h - mean (bf16 stash) or -mean
          const float shift = st.z - mean;
          const size_t rowt = static_cast<size_t>(t) * D;
          for (int c0 = 0; c0 < D; c0 += 256) {     // warp-uniform; lanes past D idle
            const int c = c0 + 8 * lane;
            const float sh = __shfl_sync(0xffffffffu, shift, (c >> 7) & 7);
            if (c >= D) continue;
            float o8[8];
            if (fp32_stash) {
              const float4 x0 = ld_global_cg_f4(a.o_save + rowt + c);
              const float4 x1 = ld_global_cg_f4(a.o_save + rowt + c + 4);
              o8[0] = x0.x; o8[1] = x0.y; o8[2] = x0.z; o8[3] = x0.w;
              o8[4] = x1.x; o8[5] = x1.y; o8[6] = x1.z; o8[7] = x1.w;
            } else {
              const uint4 w4 =
                  ld_global_cg_u4(reinterpret_cast<const __nv_bfloat16*>(a.y) + rowt + c);
              const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[i]));
                o8[2 * i] = f.x;
                o8[2 * i + 1] = f.y;
              }
            }
            const uint4 uw = __ldg(reinterpret_cast<const uint4*>(
                reinterpret_cast<const __nv_bfloat16*>(a.u) + rowt + c));
            const uint32_t uv[4] = {uw.x, uw.y, uw.z, uw.w};
            // LayerNorm weight and bias of these 8 columns (ones and zeros without tables)
            float gw[8], gb[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              gw[i] = 1.f;
              gb[i] = 0.f;
            }
            if (a.ln_weight) {
              const float4 w0 = __ldg(reinterpret_cast<const float4*>(a.ln_weight + c));
              const float4 w1 = __ldg(reinterpret_cast<const float4*>(a.ln_weight + c + 4));
              gw[0] = w0.x; gw[1] = w0.y; gw[2] = w0.z; gw[3] = w0.w;
              gw[4] = w1.x; gw[5] = w1.y; gw[6] = w1.z; gw[7] = w1.w;
            }
            if (a.ln_bias) {
              const float4 b0 = __ldg(reinterpret_cast<const float4*>(a.ln_bias + c));
              const float4 b1 = __ldg(reinterpret_cast<const float4*>(a.ln_bias + c + 4));
              gb[0] = b0.x; gb[1] = b0.y; gb[2] = b0.z; gb[3] = b0.w;
              gb[4] = b1.x; gb[5] = b1.y; gb[6] = b1.z; gb[7] = b1.w;
            }
            uint32_t yv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 uf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uv[i]));
              yv[i] = pack_bf16x2(
                  fmaf((o8[2 * i] + sh) * rstd, gw[2 * i], gb[2 * i]) * silu_gate(uf.x),
                  fmaf((o8[2 * i + 1] + sh) * rstd, gw[2 * i + 1], gb[2 * i + 1]) * silu_gate(uf.y));
            }
            *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.y) + rowt + c) =
                make_uint4(yv[0], yv[1], yv[2], yv[3]);
          }
          if (lane == 0 && a.ln_mean) {
            a.ln_mean[t] = mean;
            a.ln_rstd[t] = rstd;
          }
        }
        if (et == 0) a.item_cnt[static_cast<size_t>(b) * a.max_tiles + m] = 0u;
      }
      g += nt;
      ++j;
    }
    if (!ok) {
      set_status(a.status, kStatusTimeout);
      *abort_flag = 1;
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == kWarpS) {
    tc_fence_after();
    // Every MMA has completed once B_DONE fired; wait for it before freeing TMEM.
    if (lane == 0) mbar_wait(bar(B_DONE), 0, nullptr);
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Per-device launch state: the shared-memory opt-in is a per-device function
// attribute and the resident CTA count a per-device property; both are taken
// once per device (not inside a stream capture of a later call).  Host
// threads may launch concurrently: the values are atomics, and two threads
// that both find them unset just compute and store the same values.
struct DeviceState {
  std::atomic<int> configured[4];
  std::atomic<int> resident[4];
};
DeviceState g_state[64];

template <bool POS, bool TIME>
cudaError_t launch_variant(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                           const CUtensorMap& tv, cudaStream_t stream) {
  constexpr int var = (POS ? 1 : 0) + (TIME ? 2 : 0);
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  DeviceState& ds = g_state[dev];
  if (!ds.configured[var].load(std::memory_order_acquire)) {
    err = cudaFuncSetAttribute(hstu_fwd_bf16_sm100<POS, TIME>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    ds.configured[var].store(1, std::memory_order_release);
  }
  int resident = ds.resident[var].load(std::memory_order_acquire);
  if (resident == 0) {
    int per_sm = 0, sms = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, hstu_fwd_bf16_sm100<POS, TIME>,
                                                        kThreads, kSmemBytes);
    if (err != cudaSuccess) return err;
    err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
    resident = std::max(1, per_sm) * std::max(1, sms);
    ds.resident[var].store(resident, std::memory_order_release);
  }
  const long long nslots = static_cast<long long>((a.B + a.group - 1) / a.group) * a.group *
                           a.max_tiles * a.H;
  const long long grid = std::min<long long>(resident, nslots);
  hstu_fwd_bf16_sm100<POS, TIME><<<static_cast<unsigned>(grid), kThreads, kSmemBytes, stream>>>(
      tq, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_bf16_sm100(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                                  const CUtensorMap& tv, cudaStream_t stream) {
  if (a.B == 0 || a.max_tiles == 0) return cudaSuccess;
  if (a.H < 1 || a.H > kMaxHeads) return cudaErrorInvalidValue;
  // Work slots are numbered in 32 bits (plus one claim window of 32 and the grid).
  if (a.group < 1 || a.group > a.B) return cudaErrorInvalidValue;
  if ((static_cast<long long>(a.B) + a.group) * a.max_tiles * a.H > 0x7FFFFF00LL)
    return cudaErrorInvalidValue;
  const bool pos = a.rab_pos != nullptr, tim = a.rab_time != nullptr;
  if (pos && tim) return launch_variant<true, true>(a, tq, tk, tv, stream);
  if (pos) return launch_variant<true, false>(a, tq, tk, tv, stream);
  if (tim) return launch_variant<false, true>(a, tq, tk, tv, stream);
  return launch_variant<false, false>(a, tq, tk, tv, stream);
}

}  // namespace hstu
