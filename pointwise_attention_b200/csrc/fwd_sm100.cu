// fwd_sm100.cu -- bf16 forward of HSTU causal pointwise aggregated attention
// on sm_100a: TMA-staged Q/K/V tiles, tcgen05 MMAs with TMEM accumulators,
// a register epilogue for bias + SiLU + causal mask between the two MMAs,
// and the LayerNorm-over-heads + SiLU(U) gate fused into the store.
//
// Operation: "HSTU (Generative Recommender)" model card, Exported PyTorch,
// HSTUBlock.forward (silu(q k^T)/t, tril, attn @ v, gate by silu(u));
// relative position / time bias: "HSTU Hierarchical Sequential Transduction
// Units", §1 and §3; post-pooling normalisation then U gate: the HSTU
// reproduction note's flowchart.
//
// Work decomposition.  A work item is one (sequence b, query tile m): 128
// query rows against key tiles n = 0..m (tiles above the diagonal are skipped;
// only the diagonal tile is masked), for all H heads.  The H CTAs of a
// thread-block cluster take one head each, so the LayerNorm over the
// concatenated heads exchanges per-row statistics through distributed shared
// memory.  The kernel is persistent: the grid holds as many clusters as can
// be resident, and each cluster loops over items that its leader CTA (rank 0)
// claims from a work counter in global memory (the first one, slot c for
// cluster c, without a claim).  Items are numbered from the most expensive
// (largest m) down, so the claims form a longest-first list schedule; slots
// whose tile lies past the end of its sequence are skipped in runs of up to
// 32 per claim.  The leader claims the next item once its loads
// for the current item are issued and hands it to every CTA of the cluster
// through an 8-entry ring in shared memory.  While the epilogue normalises
// item j, the TMA and MMA warps already load and multiply item j+1.
//
// Roles (640 threads): warp 0 issues TMA (and, in the leader, claims items);
// warp 1 allocates TMEM and issues the S = Q K^T MMAs; warp 18 issues the
// O += P V MMAs; warps 2..17 form the epilogue: warp w owns TMEM lane quarter
// w%4 (rows 32*(w%4) ..) and the 32 columns (w-2)/4 of every tile.  Each warp
// stages the position-bias diagonals and key timestamps of its own 32x32
// block in a private buffer, fetched from global memory one tile ahead.  A
// tcgen05.mma instruction costs its issuing thread about 110 cycles whatever
// its N up to 128, about as long as the tensor core needs for 128x128x16, so
// the two GEMMs of a tile are issued by two threads in parallel.
//
// TMEM (512 columns): three S/P buffers [0,128) [128,256) [256,384) and O
// [384,512).  S(x) = Q K^T lands in buffer x % 3 in fp32; the epilogue writes
// P' = SiLU(S+bias) over it as packed bf16 pairs (each warp only over columns
// it has already read: its 32 keys take 16 columns), and P' is the A operand
// (from TMEM) of O' += P' V; O = O' / N in the epilogue.  S(x+3) reuses the
// buffer once P(x).V has completed; with three buffers S(x+1) and S(x+2) are
// computed while the epilogue is on tile x.
//
// Every tcgen05.ld/st is warp-collective (.sync.aligned): they are issued by
// all 32 lanes with warp-uniform control flow; only global accesses are
// predicated per row.
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"
#include "tile_math.cuh"

namespace hstu {
namespace {

constexpr int kThreads = 640;
constexpr int kEpiThreads = 512;
constexpr int kColGroups = 4;               // epilogue warpgroups, 32 columns each
constexpr int kRows = 128;                  // query rows per tile
constexpr int kCols = 128;                  // keys per tile
constexpr int kHalf = 16384;                // 128 rows x 64 bf16 (one 128B-swizzle slab)
constexpr int kTile = 2 * kHalf;            // 128 x 128 bf16
constexpr int kKStages = 3;                 // K tiles in flight (S = Q K^T needs them first)
constexpr int kVStages = 2;                 // V tiles in flight (P.V comes a tile later)
constexpr int kRing = 8;                    // claimed items handed to the cluster, in flight
constexpr int kMaxHeads = 8;

// shared-memory map (byte offsets from a 1024-aligned base)
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kTile;                    // kKStages tiles
constexpr int kOffV = kOffK + kKStages * kTile;         // kVStages tiles
// Per epilogue warp: the half position bias of the 63 diagonals its 32x32
// block touches, as 64 overlapping bf16 pairs (entry k holds diagonals k and
// k-1, the two an element pair needs), and 32 int64 key timestamps.
constexpr int kWarpStage = 64 * 4 + 32 * 8;             // bytes per warp
constexpr int kOffWarp = kOffV + kVStages * kTile;
// LayerNorm partials of the four column groups, [4][128] (sum, M2) pairs.  They
// alias the staging buffers, which are idle between an item's last tile and
// the next item's first.
constexpr int kOffLoc = kOffWarp;
constexpr int kOffThr = kOffWarp + 16 * kWarpStage;     // kThrLen int64 thresholds
constexpr int kOffFirst = kOffThr + kThrLen * 8;        // 64 int8 first bucket per octave
constexpr int kOffRabT = kOffFirst + 64;                // 128 fp32 half time-bias row
// Cluster exchange slots of the per-head row statistics: [2 item parities]
// [kMaxHeads][128 rows] (sum, M2) pairs.
constexpr int kOffRed = kOffRabT + 128 * 4;
constexpr int kRedBytes = 2 * kMaxHeads * 128 * 8;
constexpr int kOffRing = kOffRed + kRedBytes;           // kRing (m, b) pairs
constexpr int kOffBar = kOffRing + kRing * 8;           // mbarriers (8 B each)
constexpr int kNumBars = 43;
constexpr int kOffMisc = kOffBar + kNumBars * 8;        // tmem base, abort flag
constexpr int kSmemBytes = kOffMisc + 64 + 1024;        // + alignment slack
static_assert(16 * kWarpStage >= kColGroups * 128 * 8, "LayerNorm partials must fit the staging");
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

// barrier indices
constexpr int B_QFULL = 0;
constexpr int B_QEMPTY = 1;
constexpr int B_KFULL = 2;    // +K stage
constexpr int B_KEMPTY = 5;   // +K stage
constexpr int B_VFULL = 8;    // +V stage
constexpr int B_VEMPTY = 10;  // +V stage
constexpr int kSBufs = 3;     // S/P buffers in TMEM
constexpr int B_SFULL = 12;   // +buffer: S(x) computed
constexpr int B_PFULL = 15;   // +buffer: P(x) written over S(x)
constexpr int B_PVDONE = 18;  // +buffer: P(x).V completed, the buffer may be rewritten
constexpr int B_OFULL = 21;
constexpr int B_DONE = 22;    // every MMA of both issuers has completed
constexpr int B_RED = 23;     // +item parity: LayerNorm statistics of all heads arrived
constexpr int B_RFULL = 25;   // +ring slot: item written
constexpr int B_REMPTY = 33;  // +ring slot (leader only): every CTA has read the item
constexpr int B_ULOAD = 41;   // the item's U tile has landed in the LayerNorm buffer
constexpr int B_LNFREE = 42;  // the LayerNorm is done with its buffer (a V stage)
static_assert(B_LNFREE < kNumBars, "barrier count");
constexpr int kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColO = 384;
constexpr int kWarpPV = 18;   // warp of the P.V issuer

constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false, false);   // Q (K-major) x K (K-major)
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, false, true);   // P (TMEM) x V (MN-major)

__device__ __forceinline__ void set_status(int* status, int bit) {
  if (status) atomicOr(status, bit);
}

struct EpiCtx {
  const uint32_t* wpk;        // warp's half position bias pairs: element pair (lane, 2i, 2i+1)
                              // -> wpk[lane - 2i] = (diag of col 2i, diag of col 2i+1)
  const long long* kts;       // warp's 32 key timestamps
  const long long* thr;       // bucket thresholds
  const signed char* first;   // first bucket per octave
  const float* rabt;          // half time bias per bucket
  long long my_ts;            // this row's timestamp
  bool chunk_sorted;          // the warp's key timestamps are non-decreasing
  float inv_n;                // 1 / N_b
  int r;                      // row in the tile
  int lane;
};

// Time bias of a 32-column chunk for this row.  With the tile's key timestamps
// sorted and the row not before the chunk's last key, |t_i - t_j| falls along
// the chunk, so the bucket lies between the buckets k0 >= k1 of its two ends;
// when they differ by at most one, the columns before `split` (bisection) take
// k0 and the rest k1 ("simple").  Otherwise every element takes the full search.
struct ChunkTime {
  float hi, lo;     // half time bias of buckets k0 and k1
  int split;        // columns [0, split) take `hi`
  bool simple;
};

__device__ __forceinline__ ChunkTime chunk_time(const EpiCtx& e) {
  ChunkTime ct;
  ct.hi = ct.lo = 0.f;
  ct.split = 0;
  const long long d0 = e.my_ts - e.kts[0];
  const long long d1 = e.my_ts - e.kts[31];
  ct.simple = e.chunk_sorted && d1 >= 0;
  if (ct.simple) {
    const int k0 = time_bucket(d0, e.thr, e.first);
    const int k1 = time_bucket(d1, e.thr, e.first);
    ct.simple = (k0 - k1) <= 1;
    ct.hi = e.rabt[k0];
    ct.lo = e.rabt[k1];
    if (k0 != k1) {
      // columns c with t_i - t_c >= thr[k0]  <=>  t_c <= t_i - thr[k0]
      const long long lim = e.my_ts - e.thr[k0];
      int lo = 0, hi = 32;   // first column with kts > lim
#pragma unroll 1
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (e.kts[mid] <= lim) lo = mid + 1; else hi = mid;
      }
      ct.split = lo;
    }
  }
  return ct;
}

// P' = N * SiLU(S + bias) / N for two adjacent columns, packed as bf16x2:
//   hx = (S + bias)/2,  P' = hx (1 + tanh(hx)) = SiLU(S + bias).
// hx is rounded to bf16, tanh and the fused multiply-add run on bf16 pairs
// (one MUFU operation per two elements); the 1/N factor is applied to O in
// fp32 after the A.V accumulation instead of to every element of P.
__device__ __forceinline__ uint32_t p_pair(float hx0, float hx1) {
  __nv_bfloat162 h2 = __floats2bfloat162_rn(hx0, hx1);   // .x (low half) = hx0
  const uint32_t hv = *reinterpret_cast<uint32_t*>(&h2);
  uint32_t tv, pv;
  asm("tanh.approx.bf16x2 %0, %1;" : "=r"(tv) : "r"(hv));
  asm("fma.rn.bf16x2 %0, %1, %2, %1;" : "=r"(pv) : "r"(hv), "r"(tv));
  return pv;
}

// MODE 0: position bias only (or none); 1: plus a per-row time bias constant
// (`lo`); 2: plus the per-row two-value split; 3: per-element bucket search.
template <bool POS, int MODE, bool DIAG>
__device__ __forceinline__ void chunk_to_p(const uint32_t (&sraw)[32], int c0, const EpiCtx& e,
                                           const ChunkTime& ct, uint32_t (&packed)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float hx[2], hbp[2] = {0.f, 0.f};
    if (POS) {
      const uint32_t w = e.wpk[e.lane - 2 * i];
      hbp[0] = __uint_as_float(w << 16);
      hbp[1] = __uint_as_float(w & 0xFFFF0000u);
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int cl = 2 * i + hh;
      float hb = hbp[hh];
      if (MODE == 1) hb += ct.lo;
      if (MODE == 2) hb += (cl < ct.split) ? ct.hi : ct.lo;
      if (MODE == 3) hb += e.rabt[time_bucket(e.my_ts - e.kts[cl], e.thr, e.first)];
      hx[hh] = fmaf(__uint_as_float(sraw[cl]), 0.5f, hb);
    }
    uint32_t pv = p_pair(hx[0], hx[1]);
    if (DIAG) {   // causal mask: column c > row r is exactly zero
      const int c = c0 + 2 * i;
      const uint32_t keep = (c > e.r ? 0u : 0x0000FFFFu) | (c + 1 > e.r ? 0u : 0xFFFF0000u);
      pv &= keep;
    }
    packed[i] = pv;
  }
}

// Chunk k (32 columns) of this thread's 64 columns -> 16 packed P words.
template <bool POS, bool TIME, bool DIAG>
__device__ __forceinline__ void chunk_p(const uint32_t (&sv)[32], int c0, const EpiCtx& e,
                                        uint32_t (&packed)[16]) {
  if (!TIME) {
    chunk_to_p<POS, 0, DIAG>(sv, c0, e, ChunkTime{}, packed);
  } else {
    const ChunkTime ct = chunk_time(e);
    // Warp-uniform choice of the element loop.
    if (!__all_sync(0xffffffffu, ct.simple)) {
      chunk_to_p<POS, 3, DIAG>(sv, c0, e, ct, packed);
    } else if (__any_sync(0xffffffffu, ct.split != 0)) {
      chunk_to_p<POS, 2, DIAG>(sv, c0, e, ct, packed);
    } else {
      chunk_to_p<POS, 1, DIAG>(sv, c0, e, ct, packed);
    }
  }
}

// This thread's 32 columns (col0 .. col0+31) of the S tile -> P in TMEM,
// packed into columns col0 .. col0+15 of the same buffer (already read).
// `wpk` holds the warp's 64 staged diagonal pairs, `kts` its 32 key timestamps.
template <bool POS, bool TIME, bool DIAG>
__device__ __forceinline__ void chunk_to_tmem(uint32_t s_addr, int col0, EpiCtx& e,
                                              const uint32_t* wpk, const long long* kts,
                                              bool sorted) {
  uint32_t sv[32];
  uint32_t packed[16];
  tmem_ld32_nowait(s_addr + col0, sv);
  tmem_wait_ld_dep(sv);
  // element (lane, cl) uses diagonal index lane - cl + 31
  e.wpk = wpk + 31;
  e.kts = kts;
  e.chunk_sorted = sorted;
  chunk_p<POS, TIME, DIAG>(sv, col0, e, packed);
  tmem_st16(s_addr + col0, packed);
}

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
// L2 together; inside a group, slot r is the item (m = M-1 - r/G, b = group
// * G + r mod G), so the most expensive query tiles of the group come first
// (a longest-first list schedule), and the K/V tiles every query tile of a
// sequence reads stay in L2 while the group is worked on.
__device__ __forceinline__ int2 slot_item(unsigned k, unsigned G, int M) {
  const unsigned per = G * static_cast<unsigned>(M);
  const unsigned grp = k / per, r = k % per;
  return make_int2(M - 1 - static_cast<int>(r / G), static_cast<int>(grp * G + r % G));
}

// Claims this cluster's next item (warp-collective; leader CTA's warp 0).  Cluster c takes slot c as its first
// item without touching the counter (the first `base` slots, one per
// cluster); every later claim takes slot base + the counter's old value from
// an atomic add.  A slot whose tile lies past its sequence end holds no work:
// the warp then tests the 31 slots after it and raises the counter past the
// empty ones among them (atomicMax; every skipped slot was seen empty, and no
// slot is handed out twice), then claims again.  Returns (-1, -1) once the
// slots are exhausted.
template <bool POS>
__device__ int2 claim_item(const FwdArgs& a, unsigned* counter, unsigned nslots, unsigned base,
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
    if (k >= nslots) return make_int2(-1, -1);
    const unsigned slot = k + static_cast<unsigned>(lane);
    bool valid = false;
    if (slot < nslots && (!fixed || lane == 0)) {
      const int2 it = slot_item(slot, G, M);
      if (it.y < a.B) {   // the last group may be partial
        const int2 sq = load_seq(a, it.y, POS);
        if (sq.y < 0) {
          if (it.x == 0) set_status(a.status, kStatusBadOffsets);
        } else {
          valid = kRows * it.x < sq.y;
        }
      }
    }
    const unsigned vb = __ballot_sync(0xffffffffu, valid);
    if (vb & 1u) return slot_item(k, G, M);
    if (fixed) {          // the cluster's own first slot is empty: claim from the counter
      fixed = false;
      continue;
    }
    const unsigned rest = vb & ~1u;
    const unsigned skip_to = rest ? k + static_cast<unsigned>(__ffs(rest) - 1) : k + 32u;
    if (lane == 0 && skip_to > k + 1) atomicMax(counter, min(skip_to, nslots) - base);
  }
}

template <bool POS, bool TIME>
__global__ void __launch_bounds__(kThreads, 1)
    hstu_fwd_bf16_sm100(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_u,
                        const __grid_constant__ CUtensorMap tm_y,
                        const __grid_constant__ FwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int H = a.H;
  const int h = static_cast<int>(cluster_ctarank());   // head = rank in the cluster
  const bool leader = (h == 0);

  auto bar = [&](int i) { return sbase + kOffBar + 8u * i; };
  auto ring_addr = [&](int slot) { return sbase + kOffRing + 8u * slot; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  long long* s_thr = reinterpret_cast<long long*>(smem + kOffThr);
  signed char* s_first = reinterpret_cast<signed char*>(smem + kOffFirst);
  float* s_rabt = reinterpret_cast<float*>(smem + kOffRabT);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      uint32_t count = 1;
      if (i >= B_PFULL && i < B_PFULL + kSBufs) count = kEpiThreads;
      if (i == B_DONE) count = 2;                                        // both issuers
      if (i >= B_REMPTY && i < B_REMPTY + kRing) count = static_cast<uint32_t>(H);
      mbar_init(bar(i), count);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + kOffMisc, kTmemCols);
    tmem_relinquish();
  }
  if (TIME && warp >= 2 && warp < kWarpPV) {
    const int et = threadIdx.x - 64;
    for (int i = et; i < kThrLen; i += kEpiThreads) s_thr[i] = a.bt.thr[i];
    if (et < 64) s_first[et] = a.bt.first_k[et];
    if (et < a.nb) s_rabt[et] = 0.5f * __ldg(a.rab_time + static_cast<size_t>(h) * a.nb + et);
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_u);
    tma_prefetch_desc(&tm_y);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Every CTA of the cluster has initialised its barriers before any remote access.
  cluster_arrive();
  cluster_wait();
  const uint32_t tmem = misc[0];

  // Item j of this cluster sits in ring slot j % kRing; every role reads it in order.
  auto wait_item = [&](int j) -> bool {
    return mbar_wait<true>(bar(B_RFULL + j % kRing), (j / kRing) & 1, abort_flag);
  };
  auto read_item = [&](int j) -> int2 {
    int2 v;
    asm volatile("ld.shared.v2.s32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(ring_addr(j % kRing))
                 : "memory");
    return v;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    unsigned* counter = reinterpret_cast<unsigned*>(a.status) + kSchedCounterWord;
    unsigned* done = reinterpret_cast<unsigned*>(a.status) + kSchedDoneWord;
    const unsigned nslots = static_cast<unsigned>((a.B + a.group - 1) / a.group) *
                            static_cast<unsigned>(a.group) * static_cast<unsigned>(a.max_tiles);
    // Leader: claim item j and hand it to every CTA of the cluster (warp-collective).
    auto fetch = [&](int j) -> int2 {
      bool okf = true;
      int2 it = make_int2(-1, -1);
      if (leader) {
        // The slot's previous item (j - kRing) must have been read by every CTA.
        if (lane == 0 && j >= kRing)
          okf = mbar_wait<true>(bar(B_REMPTY + j % kRing), ((j / kRing) - 1) & 1, abort_flag);
        okf = __shfl_sync(0xffffffffu, okf, 0);
        if (okf) {
          const unsigned clusters = gridDim.x / static_cast<unsigned>(H);
          it = claim_item<POS>(a, counter, nslots, clusters,
                               j == 0 ? static_cast<int>(blockIdx.x / static_cast<unsigned>(H)) : -1,
                               lane);
          if (lane == 0) {
            for (int pr = 0; pr < H; ++pr) {
              st_cluster_v2_s32(mapa_shared(ring_addr(j % kRing), pr), it.x, it.y);
              mbar_arrive_cluster(mapa_shared(bar(B_RFULL + j % kRing), pr));
            }
          }
        }
      } else {
        if (lane == 0) {
          okf = wait_item(j);
          if (okf) it = read_item(j);
        }
        okf = __shfl_sync(0xffffffffu, okf, 0);
        it.x = __shfl_sync(0xffffffffu, it.x, 0);
        it.y = __shfl_sync(0xffffffffu, it.y, 0);
      }
      __syncwarp();
      return okf ? it : make_int2(-2, -2);
    };

    int k_last[kKStages] = {-1, -1, -1}, v_last[kVStages] = {-1, -1};
    int q_last = -1;
    bool ok = true;
    int j = 0, g = 0;
    int2 it = fetch(0);
    while (it.x >= 0) {
      if (lane == 0) {
        const int m = it.x, nt = m + 1;
        const int s = __ldg(a.offsets + it.y);
        if (j > 0) ok = mbar_wait(bar(B_QEMPTY), (j - 1) & 1, abort_flag);
        if (ok) {
          const int row0 = s + kRows * m;
          mbar_arrive_expect_tx(bar(B_QFULL), kTile);
          tma_load_3d(sbase + kOffQ, &tm_q, bar(B_QFULL), 0, h, row0);
          tma_load_3d(sbase + kOffQ + kHalf, &tm_q, bar(B_QFULL), 64, h, row0);
          q_last = j;
        }
        // K runs one tile ahead of V: K(x+1) is requested before V(x), whose
        // stage frees only when P(x-2).V completes.  x is the running tile index.
        auto load_k = [&](int x, int n) -> bool {
          const int st = x % kKStages, use = x / kKStages;
          if (use > 0 && !mbar_wait(bar(B_KEMPTY + st), (use - 1) & 1, abort_flag)) return false;
          const int krow = s + kCols * n;
          mbar_arrive_expect_tx(bar(B_KFULL + st), kTile);
          tma_load_3d(sbase + kOffK + st * kTile, &tm_k, bar(B_KFULL + st), 0, h, krow);
          tma_load_3d(sbase + kOffK + st * kTile + kHalf, &tm_k, bar(B_KFULL + st), 64, h, krow);
          k_last[st] = use;
          return true;
        };
        auto load_v = [&](int x, int n) -> bool {
          const int st = x % kVStages, use = x / kVStages;
          if (use > 0 && !mbar_wait(bar(B_VEMPTY + st), (use - 1) & 1, abort_flag)) return false;
          const int krow = s + kCols * n;
          mbar_arrive_expect_tx(bar(B_VFULL + st), kTile);
          tma_load_3d(sbase + kOffV + st * kTile, &tm_v, bar(B_VFULL + st), 0, h, krow);
          tma_load_3d(sbase + kOffV + st * kTile + kHalf, &tm_v, bar(B_VFULL + st), 64, h, krow);
          v_last[st] = use;
          return true;
        };
        if (ok) ok = load_k(g, 0);
        for (int n = 0; n < nt && ok; ++n) {
          if (n + 1 < nt) ok = load_k(g + n + 1, n + 1);
          // The previous item's LayerNorm borrows the V stage of this item's
          // first tile: wait until its U load and Y store are done with it.
          if (ok && n == 0 && j > 0) ok = mbar_wait(bar(B_LNFREE), (j - 1) & 1, abort_flag);
          if (ok) ok = load_v(g + n, n);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      g += it.x + 1;
      ++j;
      it = fetch(j);
    }
    if (it.x == -2) ok = false;
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
      if (leader) {
        // The last cluster to finish returns the work counter to zero for the next launch.
        __threadfence();
        const unsigned clusters = gridDim.x / static_cast<unsigned>(H);
        if (atomicAdd(done, 1u) == clusters - 1) {
          atomicExch(counter, 0u);
          atomicExch(done, 0u);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ S issuer
    if (lane == 0) {
      bool ok = true;
      int j = 0, g = 0;
      for (;;) {
        ok = wait_item(j);
        if (!ok) break;
        const int2 it = read_item(j);
        if (it.x < 0) break;
        const int nt = it.x + 1;
        ok = mbar_wait(bar(B_QFULL), j & 1, abort_flag);
        for (int n = 0; n < nt && ok; ++n) {
          const int x = g + n, st = x % kKStages, buf = x % kSBufs;
          // The buffer's previous tile x-3 has been consumed by its P.V.
          if (x >= kSBufs)
            ok = mbar_wait(bar(B_PVDONE + buf), ((x - kSBufs) / kSBufs) & 1, abort_flag);
          if (ok) ok = mbar_wait(bar(B_KFULL + st), (x / kKStages) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t d = tmem + kColS0 + 128u * buf;
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
        const int2 it = read_item(j);
        if (it.x < 0) break;
        const int nt = it.x + 1;
        for (int n = 0; n < nt && ok; ++n) {
          const int x = g + n, st = x % kVStages, buf = x % kSBufs;
          ok = mbar_wait(bar(B_PFULL + buf), (x / kSBufs) & 1, abort_flag);
          if (ok) ok = mbar_wait(bar(B_VFULL + st), (x / kVStages) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t va = sbase + kOffV + st * kTile;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            // 16 keys per step: rows 16ks.. of the V tile; the two 64-column
            // halves of d_v are 16 KB apart (leading byte offset).
            // P keys 16ks..16ks+15: column group ks/2 holds its 32 keys in 16 columns.
            mma_ts(tmem + kColO, tmem + kColS0 + 128u * buf + 32u * (ks >> 1) + 8u * (ks & 1),
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
  } else if (warp < kWarpPV) {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3;                      // TMEM lane quarter
    const int cq = (warp - 2) >> 2;               // 32-column group of the S/P and O tiles
    const int r = q4 * 32 + lane;                 // row within the tile
    const int et = threadIdx.x - 64;              // 0..511 among epilogue threads
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    const int Lw = 2 * a.L - 1;
    const int D = H * 128;
    uint8_t* wstage = smem + kOffWarp + (warp - 2) * kWarpStage;
    uint32_t* wpk = reinterpret_cast<uint32_t*>(wstage);
    long long* wts = reinterpret_cast<long long*>(wstage + 64 * 4);
    float2* loc = reinterpret_cast<float2*>(smem + kOffLoc);   // [4][128]
    float2* red = reinterpret_cast<float2*>(smem + kOffRed);   // [2][kMaxHeads][128]
    const uint32_t rempty_leader = mapa_shared(bar(B_REMPTY), 0);
    EpiCtx ec;
    ec.thr = s_thr;
    ec.first = s_first;
    ec.rabt = s_rabt;
    ec.r = r;
    ec.lane = lane;
    bool ok = true;
    int j = 0, g = 0;

    // Named barriers cannot time out, so every epilogue warp leaves the loop
    // at the same point: the decisions to stop are OR-reduced over all of them.
    for (;;) {
      const bool got = __all_sync(0xffffffffu, wait_item(j));
      const int2 it = got ? read_item(j) : make_int2(-2, -2);
      if (named_bar_or(2, kEpiThreads, !ok || it.x < 0)) {
        if (it.x == -2) ok = false;
        break;
      }
      const int m = it.x, nt = m + 1;
      const int s = __ldg(a.offsets + it.y);
      const int n_b = __ldg(a.offsets + it.y + 1) - s;
      const int i_loc = kRows * m + r;            // local row index in the sequence
      const bool row_ok = i_loc < n_b;
      const int t_row = s + (row_ok ? i_loc : 0);
      const float nrm = a.norm_len > 0 ? static_cast<float>(a.norm_len) : static_cast<float>(n_b);
      // Rows past the sequence end (never stored) take the last token's
      // timestamp: every key is then at or before them, the chunk plans stay
      // on the cheap path, and no warp drops to the per-element search.
      ec.my_ts = TIME ? a.timestamps[row_ok ? t_row : s + n_b - 1] : 0;
      ec.inv_n = 1.0f / nrm;
      // The gate input of this row is read at the end of the item: ask L2 for it now.
      if (row_ok)
        prefetch_l2(reinterpret_cast<const __nv_bfloat16*>(a.u) +
                    static_cast<size_t>(t_row) * (H * 128) + h * 128 + 32 * cq);

      // Staging of this warp's 32 x 32 block of tile n: half position bias of
      // the 63 diagonals d = r - c in [32 q4 - 32 cq - 31, 32 q4 - 32 cq + 31]
      // (table index 128 (m - n) + d + L - 1), entry k as the bf16 pair
      // (diagonal k, diagonal k-1), and the timestamps of its 32 keys (keys
      // past the sequence end repeat its last timestamp, which keeps them
      // non-decreasing; those keys are masked anyway).
      const int dbase = 32 * q4 - 32 * cq - 31;
      float pre_w0 = 0.f, pre_w1 = 0.f;
      long long pre_t = 0;
      auto prefetch = [&](int n) {
        if (POS) {
          const int t0 = kRows * (m - n) + dbase + lane + a.L - 1;
          const float* tab = a.rab_pos + static_cast<size_t>(h) * Lw;
          pre_w0 = (t0 >= 0 && t0 < Lw) ? __ldg(tab + t0) : 0.f;
          pre_w1 = (lane < 31 && t0 + 32 >= 0 && t0 + 32 < Lw) ? __ldg(tab + t0 + 32) : 0.f;
        }
        if (TIME) {
          const int jj = kCols * n + 32 * cq + lane;
          pre_t = a.timestamps[s + (jj < n_b ? jj : n_b - 1)];
        }
      };
      bool sorted = true;
      auto stage = [&]() {   // previous users of the buffer (this warp) are done
        if (POS) {
          const float v0 = 0.5f * pre_w0, v1 = 0.5f * pre_w1;
          float p0 = __shfl_up_sync(0xffffffffu, v0, 1);
          float p1 = __shfl_up_sync(0xffffffffu, v1, 1);
          const float e0 = __shfl_sync(0xffffffffu, v0, 31);
          if (lane == 0) {
            p0 = 0.f;
            p1 = e0;
          }
          __nv_bfloat162 b0 = __floats2bfloat162_rn(v0, p0);   // .x (low) = diagonal k
          __nv_bfloat162 b1 = __floats2bfloat162_rn(v1, p1);
          wpk[lane] = *reinterpret_cast<uint32_t*>(&b0);
          wpk[32 + lane] = *reinterpret_cast<uint32_t*>(&b1);
        }
        if (TIME) {
          wts[lane] = pre_t;
          const long long nx = __shfl_down_sync(0xffffffffu, pre_t, 1);
          sorted = !__any_sync(0xffffffffu, lane < 31 && nx < pre_t);
        }
        __syncwarp();
      };

      prefetch(0);
      stage();
      for (int n = 0; n < nt; ++n) {
        const int x = g + n, buf = x % kSBufs;
        if (n + 1 < nt) prefetch(n + 1);          // global loads overlap this tile
        if (ok) ok = mbar_wait(bar(B_SFULL + buf), (x / kSBufs) & 1, abort_flag);
        // The TMEM loads/stores below are warp-collective: keep the decision warp-uniform.
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;                           // on to the collective exit below
        tc_fence_after();
        const uint32_t s_addr = tmem + lane_addr + kColS0 + 128u * buf;
        if (n == m)
          chunk_to_tmem<POS, TIME, true>(s_addr, 32 * cq, ec, wpk, wts, sorted);
        else
          chunk_to_tmem<POS, TIME, false>(s_addr, 32 * cq, ec, wpk, wts, sorted);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_PFULL + buf));
        if (n + 1 < nt) stage();
      }

      // -------------------------------------------- LayerNorm over heads + gate
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_OFULL), j & 1, abort_flag));
      if (ok) tc_fence_after();
      // The row's 32 values of this head and column quarter stay in registers.
      float ov[32];
      {
        uint32_t o0[32];
        if (ok) {
          tmem_ld32_nowait(tmem + lane_addr + kColO + 32u * cq, o0);
          tmem_wait_ld_dep(o0);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o0[i] = 0u;
        }
        // O accumulated SiLU(.) terms: apply 1/N here, in fp32.
#pragma unroll
        for (int i = 0; i < 32; ++i) ov[i] = __uint_as_float(o0[i]) * ec.inv_n;
      }
      const size_t rowD = static_cast<size_t>(t_row) * D + static_cast<size_t>(h) * 128 + 32 * cq;
      // U and Y of the item travel by TMA through the V stage of the next
      // item's first tile (every P.V of this item has completed; the producer
      // waits for B_LNFREE before loading it again).  In that 128B-swizzled
      // tile, 16-byte chunk c of row r sits at r * 128 + 16 (c ^ (r % 8)) of
      // its 64-column half: a warp's 32 rows hit every bank once per 8 rows.
      const uint32_t lnbuf = sbase + kOffV + ((g + nt) % kVStages) * kTile;
      if (et == 0) {
        const int row0 = s + kRows * m;
        mbar_arrive_expect_tx(bar(B_ULOAD), kTile);
        tma_load_3d(lnbuf, &tm_u, bar(B_ULOAD), 0, h, row0);
        tma_load_3d(lnbuf + kHalf, &tm_u, bar(B_ULOAD), 64, h, row0);
      }
      const uint32_t myrow = lnbuf + (cq >> 1) * kHalf + r * 128;
      auto chunk_addr = [&](int i) {   // i-th 16-byte chunk of this thread's 32 columns
        return myrow + 16u * static_cast<uint32_t>((4 * (cq & 1) + i) ^ (r & 7));
      };
      if (ok && row_ok && a.o_save) {
        float* od = a.o_save + rowD;
        if (a.vec32) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t w[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) w[q] = __float_as_uint(ov[8 * i + q]);
            st_global_v8(od + 8 * i, w);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            reinterpret_cast<float4*>(od)[i] =
                make_float4(ov[4 * i], ov[4 * i + 1], ov[4 * i + 2], ov[4 * i + 3]);
        }
      }
      // Row statistics of the 32 values: sum and sum of squared deviations.
      {
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
      tc_fence_before();
      if (named_bar_or(1, kEpiThreads, !ok)) {
        ok = false;
        break;
      }
      // Every role of this CTA has read item j: release its ring slot.
      if (et == 0) mbar_arrive_cluster(rempty_leader + 8u * (j % kRing));
      const int pj = j & 1;
      if (cq == 0) {
        // Combine the four 32-column groups (equal counts) into this head's
        // (sum, M2) and send it to every CTA of the cluster.
        const float2 p0 = loc[r], p1 = loc[128 + r], p2 = loc[256 + r], p3 = loc[384 + r];
        const float hs = (p0.x + p1.x) + (p2.x + p3.x);
        const float mh = hs * (1.0f / 128.0f);
        const float e0 = p0.x * (1.0f / 32.0f) - mh, e1 = p1.x * (1.0f / 32.0f) - mh;
        const float e2 = p2.x * (1.0f / 32.0f) - mh, e3 = p3.x * (1.0f / 32.0f) - mh;
        const float hm2 = (p0.y + p1.y) + (p2.y + p3.y) +
                          32.0f * ((e0 * e0 + e1 * e1) + (e2 * e2 + e3 * e3));
        const uint32_t slot = smem_u32(red + (pj * kMaxHeads + h) * 128 + r);
        for (int pr = 0; pr < H; ++pr)
          st_async_v2_f32(mapa_shared(slot, pr), hs, hm2, mapa_shared(bar(B_RED + pj), pr));
      }
      if (et == 0) mbar_arrive_expect_tx(bar(B_RED + pj), static_cast<uint32_t>(H * 128 * 8));
      // Gate values while the statistics travel.
      if (!mbar_wait(bar(B_ULOAD), j & 1, abort_flag)) set_status(a.status, kStatusTimeout);
      float gate[32];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 ui = ld_shared_v4(chunk_addr(i));
        const __nv_bfloat162* u2 = reinterpret_cast<const __nv_bfloat162*>(&ui);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 uf = __bfloat1622float2(u2[q]);
          gate[8 * i + 2 * q] = silu_gate(uf.x);
          gate[8 * i + 2 * q + 1] = silu_gate(uf.y);
        }
      }
      if (!mbar_wait<true>(bar(B_RED + pj), (j >> 1) & 1, nullptr)) set_status(a.status, kStatusTimeout);
      // Chan's combination of the H per-head (sum, M2) pairs of 128 values each.
      const float2* rr = red + pj * kMaxHeads * 128 + r;
      float tot = 0.f;
      for (int k = 0; k < H; ++k) tot += rr[k * 128].x;
      const float mean = tot / static_cast<float>(D);
      float m2 = 0.f;
      for (int k = 0; k < H; ++k) {
        const float2 pk = rr[k * 128];
        const float dk = pk.x * (1.0f / 128.0f) - mean;
        m2 += pk.y + 128.0f * dk * dk;
      }
      const float var = m2 / static_cast<float>(D);
      const float rstd = 1.0f / sqrtf(var + a.eps);
      {
        uint32_t yw[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          __nv_bfloat162 pr = __floats2bfloat162_rn((ov[2 * q] - mean) * rstd * gate[2 * q],
                                                    (ov[2 * q + 1] - mean) * rstd * gate[2 * q + 1]);
          yw[q] = *reinterpret_cast<uint32_t*>(&pr);
        }
        // A tile whose 128 rows all belong to the sequence leaves by one TMA
        // store; the last, partial tile of a sequence stores its rows directly.
        const bool full = kRows * m + kRows <= n_b;
        if (full) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            st_shared_v4(chunk_addr(i), make_uint4(yw[4 * i], yw[4 * i + 1], yw[4 * i + 2],
                                                   yw[4 * i + 3]));
          fence_proxy_async_smem();
        } else if (row_ok) {
          __nv_bfloat16* yd = reinterpret_cast<__nv_bfloat16*>(a.y) + rowD;
          if (a.vec32) {
            st_global_v8(yd, reinterpret_cast<const uint32_t(&)[8]>(yw[0]));
            st_global_v8(yd + 16, reinterpret_cast<const uint32_t(&)[8]>(yw[8]));
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              reinterpret_cast<uint4*>(yd)[i] =
                  make_uint4(yw[4 * i], yw[4 * i + 1], yw[4 * i + 2], yw[4 * i + 3]);
          }
        }
        if (row_ok && h == 0 && cq == 0 && a.ln_mean) {
          a.ln_mean[t_row] = mean;
          a.ln_rstd[t_row] = rstd;
        }
        // Every thread is done with the buffer (its U read, its Y written).
        named_bar_sync(3, kEpiThreads);
        if (et == 0) {
          if (full) {
            tma_store_3d(&tm_y, lnbuf, 0, h, s + kRows * m);
            tma_store_3d(&tm_y, lnbuf + kHalf, 64, h, s + kRows * m);
            bulk_commit_group();
            bulk_wait_group_read0();
          }
          mbar_arrive(bar(B_LNFREE));
        }
      }
      g += nt;
      ++j;
    }
    if (!ok) {
      set_status(a.status, kStatusTimeout);
      *abort_flag = 1;
    }
    if (et == 0) bulk_wait_group0();   // the last Y stores have landed
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    // Every MMA has completed once B_DONE fired; wait for it before freeing TMEM.
    if (lane == 0) mbar_wait(bar(B_DONE), 0, nullptr);
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
  // No CTA leaves while another may still write into its shared memory.
  cluster_arrive();
  cluster_wait();
}

template <bool POS, bool TIME>
cudaError_t launch_variant(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                           const CUtensorMap& tv, const CUtensorMap& tu, const CUtensorMap& ty,
                           cudaStream_t stream) {
  // The shared-memory opt-in is a per-device function attribute, and the
  // number of co-resident clusters a per-device, per-cluster-size property:
  // both are taken once per device (not inside a stream capture of a later call).
  static bool configured[64] = {};
  static int max_clusters[64][kMaxHeads + 1] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    err = cudaFuncSetAttribute(hstu_fwd_bf16_sm100<POS, TIME>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    configured[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(a.H);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int& resident = max_clusters[dev][a.H];
  if (resident == 0) {
    cfg.gridDim = dim3(static_cast<unsigned>(a.H), 1, 1);
    int n = 0;
    err = cudaOccupancyMaxActiveClusters(&n, hstu_fwd_bf16_sm100<POS, TIME>, &cfg);
    if (err != cudaSuccess) return err;
    resident = n > 0 ? n : 1;
  }
  const long long nslots = static_cast<long long>((a.B + a.group - 1) / a.group) * a.group *
                           a.max_tiles;
  const long long clusters = std::min<long long>(resident, nslots);
  cfg.gridDim = dim3(static_cast<unsigned>(clusters * a.H), 1, 1);
  return cudaLaunchKernelEx(&cfg, hstu_fwd_bf16_sm100<POS, TIME>, tq, tk, tv, tu, ty, a);
}

}  // namespace

cudaError_t launch_fwd_bf16_sm100(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                                  const CUtensorMap& tv, const CUtensorMap& tu,
                                  const CUtensorMap& ty, cudaStream_t stream) {
  if (a.B == 0 || a.max_tiles == 0) return cudaSuccess;
  if (a.H < 1 || a.H > kMaxHeads) return cudaErrorInvalidValue;
  // Work slots are numbered in 32 bits (plus one claim window of 32).
  if (a.group < 1 || a.group > a.B) return cudaErrorInvalidValue;
  if ((static_cast<long long>(a.B) + a.group) * a.max_tiles > 0x7FFFFF00LL)
    return cudaErrorInvalidValue;
  const bool pos = a.rab_pos != nullptr, tim = a.rab_time != nullptr;
  if (pos && tim) return launch_variant<true, true>(a, tq, tk, tv, tu, ty, stream);
  if (pos) return launch_variant<true, false>(a, tq, tk, tv, tu, ty, stream);
  if (tim) return launch_variant<false, true>(a, tq, tk, tv, tu, ty, stream);
  return launch_variant<false, false>(a, tq, tk, tv, tu, ty, stream);
}

}  // namespace hstu
