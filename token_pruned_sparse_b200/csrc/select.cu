// Active-set selection and stream compaction:
//   lipar_select   (threshold / top-k)     [LIPAR] 2.B: a token whose change is
//                                          below tau is redundant and pruned.
//   lipar_group    (HSA rank split)        [HSA] 2.1: tokens partitioned into K
//                                          groups by relative-L1 velocity change.
//   lipar_schedule (HSA per-step set)      [HSA] 2.1: group k active iff
//                                          i mod (T/s_k) == 0; 2.4: first/last
//                                          m steps run every token.
//
// Design (HBM/latency-bound, N ~ 1e4..1e6):
//   * Scores map to order-preserving uint32 keys (NaN lowest, -0 == +0).
//   * Top-k / rank cuts use an MSB-first radix select, 8-bit digits, one
//     launch per digit. Each block builds a shared-memory histogram and adds it
//     to a global one; the last block to finish (atomic ticket, no spinning)
//     picks the digit bucket and resets the histogram for the next pass. After
//     four passes the exact k-th key K* and the number of ties at K* still to
//     take (krem) are known.
//   * Compaction: a count kernel writes per-block counts and its last block
//     turns them into exclusive offsets (and the device-side total); a write
//     kernel recomputes each element's class, ranks it with warp ballots and
//     popc, and writes the ascending index list. Ties at K* are taken in index
//     order, so the result is unique.
#include <mutex>

#include "trace.cuh"
#include "tps_internal.cuh"

namespace tps {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kItems = 4;
constexpr int kTile = kThreads * kItems;  // elements per compaction block
constexpr int kMaxBound = 7;              // rank cuts (K <= 8 groups)

struct SelHdr {
  unsigned int ticket;     // last-block ticket of the count kernels
  unsigned int ticket_r;   // last-block ticket of the radix passes
  unsigned int pad[2];
  unsigned int prefix[8];  // radix prefix, finally K*, per cut
  unsigned int krem[8];    // ties at K* still to take, per cut
  unsigned int hist[kMaxBound][256];
};
constexpr size_t kHdrBytes = (sizeof(SelHdr) + 255) / 256 * 256;

struct Cuts {
  unsigned int k[kMaxBound];
};

inline int64_t n_blocks(int64_t N) { return (N + kTile - 1) / kTile; }

__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t b = __float_as_uint(s);
  if ((b & 0x7fffffffu) > 0x7f800000u) return 0u;  // NaN ranks below everything
  if (b == 0x80000000u) b = 0u;                    // -0 equals +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Inclusive scan of one value per thread over the 256-thread block.
__device__ __forceinline__ unsigned int block_incl_scan(unsigned int v, unsigned int* total) {
  __shared__ unsigned int wsum[kWarps];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  unsigned int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[w] = x;
  __syncthreads();
  unsigned int add = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < kWarps; ++i) {
    const unsigned int s = wsum[i];
    add += (i < w) ? s : 0u;
    tot += s;
  }
  __syncthreads();
  *total = tot;
  return x + add;
}

__device__ __forceinline__ unsigned int block_sum(unsigned int v) {
  unsigned int tot;
  block_incl_scan(v, &tot);
  return tot;
}

// True in every thread of the block that finished last (after all others
// published their results with a fence). No thread ever waits on another block.
__device__ __forceinline__ bool last_block(unsigned int* ticket) {
  __shared__ bool s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (s_last) __threadfence();
  return s_last;
}

// ---- radix select -------------------------------------------------------------
__global__ void sel_init(SelHdr* h, int nbound, Cuts cuts) {
  for (int i = threadIdx.x; i < kMaxBound * 256; i += blockDim.x) (&h->hist[0][0])[i] = 0u;
  if (threadIdx.x < 8) {
    h->prefix[threadIdx.x] = 0u;
    h->krem[threadIdx.x] = threadIdx.x < nbound ? cuts.k[threadIdx.x] : 0u;
  }
  if (threadIdx.x == 0) {
    h->ticket = 0u;
    h->ticket_r = 0u;
  }
}

// One 8-bit digit (bits [shift, shift+8)) for every cut at once.
__global__ void __launch_bounds__(kThreads) radix_pass(const float* __restrict__ s, int64_t N,
                                                       SelHdr* h, int nbound, int shift) {
  __shared__ unsigned int sh[kMaxBound][256];
  for (int i = threadIdx.x; i < nbound * 256; i += kThreads) (&sh[0][0])[i] = 0u;
  const unsigned int himask = shift >= 24 ? 0u : (0xffffffffu << (shift + 8));
  unsigned int pre[kMaxBound];
#pragma unroll
  for (int b = 0; b < kMaxBound; ++b) pre[b] = b < nbound ? h->prefix[b] : 0u;
  __syncthreads();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t n = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; n < N; n += stride) {
    const unsigned int key = score_key(s[n]);
    const unsigned int dig = (key >> shift) & 255u;
#pragma unroll
    for (int b = 0; b < kMaxBound; ++b)
      if (b < nbound && (key & himask) == pre[b]) atomicAdd(&sh[b][dig], 1u);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nbound * 256; i += kThreads) {
    const unsigned int v = (&sh[0][0])[i];
    if (v) atomicAdd(&(&h->hist[0][0])[i], v);
  }
  if (!last_block(&h->ticket_r)) return;
  // Last block: for each cut, thread t looks at bucket 255 - t (descending).
  for (int b = 0; b < nbound; ++b) {
    const unsigned int need = __ldcg(&h->krem[b]);
    const int bin = 255 - threadIdx.x;
    const unsigned int c = __ldcg(&h->hist[b][bin]);
    unsigned int tot;
    const unsigned int incl = block_incl_scan(c, &tot);
    const unsigned int excl = incl - c;
    if (need > 0 && excl < need && incl >= need) {
      h->prefix[b] = pre[b] | (static_cast<unsigned int>(bin) << shift);
      h->krem[b] = need - excl;
    }
    h->hist[b][bin] = 0u;
  }
  if (threadIdx.x == 0) h->ticket_r = 0u;
}

// ---- element classes ----------------------------------------------------------
// 0 = not selected, 1 = selected, 2 = tie at K* (selected in index order while
// fewer than krem ties have been taken).
struct ThreshCls {
  const float* s;
  float tau;
  __device__ __forceinline__ int operator()(int64_t n, const SelHdr*) const {
    return s[n] >= tau ? 1 : 0;
  }
};
struct TopkCls {
  const float* s;
  __device__ __forceinline__ int operator()(int64_t n, const SelHdr* h) const {
    const unsigned int key = score_key(s[n]);
    const unsigned int ks = h->prefix[0];
    return key > ks ? 1 : (key == ks ? 2 : 0);
  }
};
struct SchedCls {
  const int8_t* g;
  unsigned int act;  // bit k set: group k active this step
  int K;
  __device__ __forceinline__ int operator()(int64_t n, const SelHdr*) const {
    const int v = g[n];
    return (v >= 0 && v < K && ((act >> v) & 1u)) ? 1 : 0;
  }
};

// Per-block counts (column 0: selected, column 1: ties), then in the last
// block: exclusive offsets per column and the device-side total.
template <class Cls>
__global__ void __launch_bounds__(kThreads) compact_count(Cls cls, int64_t N, SelHdr* h,
                                                          unsigned int* cnt, unsigned int* off,
                                                          int ncol, int32_t* count_out) {
  const int64_t nb = gridDim.x;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kTile;
  unsigned int sel = 0, tie = 0;
#pragma unroll
  for (int it = 0; it < kItems; ++it) {
    const int64_t n = base + it * kThreads + threadIdx.x;
    if (n < N) {
      const int c = cls(n, h);
      sel += c == 1;
      tie += c == 2;
    }
  }
  sel = block_sum(sel);
  if (ncol > 1) tie = block_sum(tie);
  if (threadIdx.x == 0) {
    cnt[blockIdx.x] = sel;
    if (ncol > 1) cnt[nb + blockIdx.x] = tie;
  }
  if (!last_block(&h->ticket)) return;
  unsigned int totals[2] = {0u, 0u};
  for (int col = 0; col < ncol; ++col) {
    unsigned int run = 0;
    for (int64_t i0 = 0; i0 < nb; i0 += kThreads) {
      const int64_t i = i0 + threadIdx.x;
      const unsigned int v = i < nb ? __ldcg(&cnt[col * nb + i]) : 0u;
      unsigned int tot;
      const unsigned int incl = block_incl_scan(v, &tot);
      if (i < nb) off[col * nb + i] = run + incl - v;
      run += tot;
    }
    totals[col] = run;
  }
  if (threadIdx.x == 0) {
    unsigned int total = totals[0];
    if (ncol > 1) {
      const unsigned int kr = __ldcg(&h->krem[0]);
      total += totals[1] < kr ? totals[1] : kr;
    }
    if (count_out) *count_out = static_cast<int32_t>(total);
    h->ticket = 0u;
  }
}

template <class Cls>
__global__ void __launch_bounds__(kThreads) compact_write(Cls cls, int64_t N, const SelHdr* h,
                                                          const unsigned int* off, int ncol,
                                                          int32_t* __restrict__ idx) {
  __shared__ unsigned int s_sel[kWarps], s_tie[kWarps];
  const int64_t nb = gridDim.x;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kTile + w * (32 * kItems);
  unsigned int msel[kItems], mtie[kItems];
  unsigned int wsel = 0, wtie = 0;
#pragma unroll
  for (int it = 0; it < kItems; ++it) {
    const int64_t n = base + it * 32 + lane;
    const int c = n < N ? cls(n, h) : 0;
    msel[it] = __ballot_sync(0xffffffffu, c == 1);
    mtie[it] = __ballot_sync(0xffffffffu, c == 2);
    wsel += __popc(msel[it]);
    wtie += __popc(mtie[it]);
  }
  if (lane == 0) {
    s_sel[w] = wsel;
    s_tie[w] = wtie;
  }
  __syncthreads();
  unsigned int sb = off[blockIdx.x], tb = ncol > 1 ? off[nb + blockIdx.x] : 0u;
  for (int i = 0; i < w; ++i) {
    sb += s_sel[i];
    tb += s_tie[i];
  }
  const unsigned int krem = ncol > 1 ? h->krem[0] : 0u;
  const unsigned int lt = (1u << lane) - 1u;
#pragma unroll
  for (int it = 0; it < kItems; ++it) {
    const int64_t n = base + it * 32 + lane;
    const unsigned int sr = sb + __popc(msel[it] & lt);
    const unsigned int tr = tb + __popc(mtie[it] & lt);
    if ((msel[it] >> lane) & 1u) idx[sr + (tr < krem ? tr : krem)] = static_cast<int32_t>(n);
    else if (((mtie[it] >> lane) & 1u) && tr < krem) idx[sr + tr] = static_cast<int32_t>(n);
    sb += __popc(msel[it]);
    tb += __popc(mtie[it]);
  }
}

// ---- HSA group split -----------------------------------------------------------
// Per-block tie counts for every cut; the last block turns them into offsets.
__global__ void __launch_bounds__(kThreads) group_count(const float* __restrict__ s, int64_t N,
                                                        SelHdr* h, int nbound, unsigned int* cnt,
                                                        unsigned int* off) {
  const int64_t nb = gridDim.x;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kTile;
  unsigned int ks[kMaxBound];
  unsigned int eq[kMaxBound];
#pragma unroll
  for (int b = 0; b < kMaxBound; ++b) {
    ks[b] = b < nbound ? h->prefix[b] : 0u;
    eq[b] = 0u;
  }
#pragma unroll
  for (int it = 0; it < kItems; ++it) {
    const int64_t n = base + it * kThreads + threadIdx.x;
    if (n < N) {
      const unsigned int key = score_key(s[n]);
#pragma unroll
      for (int b = 0; b < kMaxBound; ++b) eq[b] += (b < nbound && key == ks[b]) ? 1u : 0u;
    }
  }
  for (int b = 0; b < nbound; ++b) {
    const unsigned int t = block_sum(eq[b]);
    if (threadIdx.x == 0) cnt[b * nb + blockIdx.x] = t;
  }
  if (!last_block(&h->ticket)) return;
  for (int b = 0; b < nbound; ++b) {
    unsigned int run = 0;
    for (int64_t i0 = 0; i0 < nb; i0 += kThreads) {
      const int64_t i = i0 + threadIdx.x;
      const unsigned int v = i < nb ? __ldcg(&cnt[b * nb + i]) : 0u;
      unsigned int tot;
      const unsigned int incl = block_incl_scan(v, &tot);
      if (i < nb) off[b * nb + i] = run + incl - v;
      run += tot;
    }
  }
  if (threadIdx.x == 0) h->ticket = 0u;
}

// group[n] = number of cuts the token does not make it above.
__global__ void __launch_bounds__(kThreads) group_write(const float* __restrict__ s, int64_t N,
                                                        const SelHdr* h, int nbound,
                                                        const unsigned int* off,
                                                        int8_t* __restrict__ group) {
  __shared__ unsigned int s_eq[kMaxBound][kWarps];
  const int64_t nb = gridDim.x;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kTile + w * (32 * kItems);
  unsigned int key[kItems];
#pragma unroll
  for (int it = 0; it < kItems; ++it) {
    const int64_t n = base + it * 32 + lane;
    key[it] = n < N ? score_key(s[n]) : 0u;
  }
  int grp[kItems] = {0, 0, 0, 0};
  const unsigned int lt = (1u << lane) - 1u;
  for (int b = 0; b < nbound; ++b) {
    const unsigned int ks = h->prefix[b];
    const unsigned int kr = h->krem[b];
    unsigned int m[kItems];
    unsigned int weq = 0;
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
      const int64_t n = base + it * 32 + lane;
      m[it] = __ballot_sync(0xffffffffu, n < N && key[it] == ks);
      weq += __popc(m[it]);
    }
    if (lane == 0) s_eq[b][w] = weq;
    __syncthreads();
    unsigned int eb = off[b * nb + blockIdx.x];
    for (int i = 0; i < w; ++i) eb += s_eq[b][i];
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
      const unsigned int r = eb + __popc(m[it] & lt);
      const bool above = key[it] > ks || (key[it] == ks && r < kr);
      grp[it] += above ? 0 : 1;
      eb += __popc(m[it]);
    }
  }
#pragma unroll
  for (int it = 0; it < kItems; ++it) {
    const int64_t n = base + it * 32 + lane;
    if (n < N) group[n] = static_cast<int8_t>(grp[it]);
  }
}

// ---- single-launch cooperative path (threshold, top-k, schedule) ----------------------
// For N up to 256 blocks of 2048 elements the whole selection runs as ONE
// cooperative launch (all blocks co-resident, guaranteed by the launch): each
// block keeps its 2048 keys in registers; the four radix passes and the final
// compaction are separated by grid barriers. A barrier is a counter in the
// workspace (zeroed before the launch) that thread 0 of every block increments
// and then polls; each poll loop is bounded by clock64 and, if it expires, sets
// the device status word (TPS_ERR_TIMEOUT) and the block leaves without
// writing results.
constexpr int kCoopItems = 8;
constexpr int kCoopTile = kThreads * kCoopItems;   // elements per block
constexpr int kCoopMaxBlocks = 256;
constexpr long long kGridWaitCycles = 2000000000LL; // ~1 s
constexpr int kCoopHdrWords = 64;                   // barrier counter + padding

enum CoopMode { kCoopThresh = 0, kCoopTopk = 1, kCoopSched = 2 };

struct CoopArgs {
  const float* s;
  float tau;
  const int8_t* g;
  unsigned int act;
  int K;
  unsigned int k;          // top-k target (>= 1)
};

inline int64_t coop_blocks(int64_t N) { return (N + kCoopTile - 1) / kCoopTile; }
// Workspace: header (barrier counter), one 256-bin histogram per radix pass
// (summed with atomics; zeroed together with the header before the launch),
// then two counts per block.
constexpr int kCoopZeroWords = kCoopHdrWords + 4 * 256;
inline size_t coop_bytes(int64_t N, int mode) {
  (void)mode;
  return kCoopZeroWords * 4 + coop_blocks(N) * 2 * 4;
}

__device__ __forceinline__ bool grid_sync(unsigned int* bar, unsigned int target, unsigned int* status,
                                          volatile int* s_fail) {
  __syncthreads();
  if (threadIdx.x == 0 && !*s_fail) {
    __threadfence();
    atomicAdd(bar, 1u);
    const long long t0 = clock64();
    while (*reinterpret_cast<volatile unsigned int*>(bar) < target) {
      if (clock64() - t0 > kGridWaitCycles) {
        *s_fail = 1;
        raise_status(status, STATUS_TIMEOUT);
        break;
      }
    }
    __threadfence();
  }
  __syncthreads();
  return *s_fail == 0;
}

template <int kMode>
__global__ void __launch_bounds__(kThreads) select_coop(CoopArgs a, int64_t N, unsigned int* ws,
                                                        int32_t* __restrict__ idx, int32_t* __restrict__ count,
                                                        unsigned int* status) {
  __shared__ unsigned int sh[256];
  __shared__ unsigned int s_pref, s_krem;
  __shared__ volatile int s_fail;
  __shared__ unsigned int s_sel[kWarps], s_tie[kWarps];
  const unsigned int G = gridDim.x, b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  unsigned int* bar = ws;
  unsigned int* hist = ws + kCoopHdrWords;                       // [4][256], top-k only
  unsigned int* cnt = ws + kCoopZeroWords;                       // [G][2]
  if (tid == 0) s_fail = 0;
  const int64_t base = static_cast<int64_t>(b) * kCoopTile + w * (32 * kCoopItems);
  uint32_t key[kCoopItems];
  int cls[kCoopItems];
#pragma unroll
  for (int it = 0; it < kCoopItems; ++it) {
    const int64_t n = base + it * 32 + lane;
    key[it] = 0u;
    cls[it] = 0;
    if (n < N) {
      if (kMode == kCoopTopk) key[it] = score_key(a.s[n]);
      else if (kMode == kCoopThresh) cls[it] = a.s[n] >= a.tau ? 1 : 0;
      else {
        const int v = a.g[n];
        cls[it] = (v >= 0 && v < a.K && ((a.act >> v) & 1u)) ? 1 : 0;
      }
    }
  }
  unsigned int nbar = 0;
  unsigned int krem = 0;
  if (kMode == kCoopTopk) {
    unsigned int prefix = 0;
    krem = a.k;
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      const unsigned int himask = pass == 0 ? 0u : (0xffffffffu << (shift + 8));
      sh[tid] = 0u;
      __syncthreads();
#pragma unroll
      for (int it = 0; it < kCoopItems; ++it) {
        const int64_t n = base + it * 32 + lane;
        if (n < N && (key[it] & himask) == prefix) atomicAdd(&sh[(key[it] >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (sh[tid]) atomicAdd(&hist[pass * 256u + tid], sh[tid]);   // one global histogram per pass
      if (!grid_sync(bar, ++nbar * G, status, &s_fail)) return;
      const int bin = 255 - tid;                                  // descending buckets
      const unsigned int c = __ldcg(&hist[pass * 256u + bin]);
      unsigned int tot;
      const unsigned int incl = block_incl_scan(c, &tot);
      const unsigned int excl = incl - c;
      if (excl < krem && incl >= krem) {
        s_pref = prefix | (static_cast<unsigned int>(bin) << shift);
        s_krem = krem - excl;
      }
      __syncthreads();
      prefix = s_pref;
      krem = s_krem;
      __syncthreads();
    }
#pragma unroll
    for (int it = 0; it < kCoopItems; ++it) {
      const int64_t n = base + it * 32 + lane;
      cls[it] = n >= N ? 0 : (key[it] > prefix ? 1 : (key[it] == prefix ? 2 : 0));
    }
  }
  // ---- compaction ------------------------------------------------------------------
  unsigned int msel[kCoopItems], mtie[kCoopItems];
  unsigned int wsel = 0, wtie = 0;
#pragma unroll
  for (int it = 0; it < kCoopItems; ++it) {
    msel[it] = __ballot_sync(0xffffffffu, cls[it] == 1);
    mtie[it] = __ballot_sync(0xffffffffu, cls[it] == 2);
    wsel += __popc(msel[it]);
    wtie += __popc(mtie[it]);
  }
  if (lane == 0) {
    s_sel[w] = wsel;
    s_tie[w] = wtie;
  }
  __syncthreads();
  if (tid == 0) {
    unsigned int bs = 0, bt = 0;
    for (int i = 0; i < kWarps; ++i) {
      bs += s_sel[i];
      bt += s_tie[i];
    }
    cnt[2 * b] = bs;
    cnt[2 * b + 1] = bt;
  }
  if (!grid_sync(bar, ++nbar * G, status, &s_fail)) return;
  // offsets of this block: sums over the blocks before it; the last block also
  // writes the device-side total
  unsigned int ps = 0, pt = 0, as = 0, at = 0;
  for (unsigned int g = tid; g < G; g += kThreads) {
    const unsigned int cs = __ldcg(&cnt[2 * g]), ct = __ldcg(&cnt[2 * g + 1]);
    if (g < b) {
      ps += cs;
      pt += ct;
    }
    as += cs;
    at += ct;
  }
  ps = block_sum(ps);
  pt = block_sum(pt);
  as = block_sum(as);
  at = block_sum(at);
  if (b == G - 1 && tid == 0) *count = static_cast<int32_t>(as + (at < krem ? at : krem));
  unsigned int sb = ps, tb = pt;
  for (int i = 0; i < w; ++i) {
    sb += s_sel[i];
    tb += s_tie[i];
  }
  const unsigned int lt = (1u << lane) - 1u;
#pragma unroll
  for (int it = 0; it < kCoopItems; ++it) {
    const int64_t n = base + it * 32 + lane;
    const unsigned int sr = sb + __popc(msel[it] & lt);
    const unsigned int tr = tb + __popc(mtie[it] & lt);
    if ((msel[it] >> lane) & 1u) idx[sr + (tr < krem ? tr : krem)] = static_cast<int32_t>(n);
    else if (((mtie[it] >> lane) & 1u) && tr < krem) idx[sr + tr] = static_cast<int32_t>(n);
    sb += __popc(msel[it]);
    tb += __popc(mtie[it]);
  }
}

// Max co-resident blocks of a cooperative kernel on the current device (cached).
template <int kMode>
int coop_capacity() {
  static std::atomic<int> cap[64];   // per device; two threads may both compute it, to the same value
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int c = cap[dev].load(std::memory_order_relaxed);
  if (!c) {
    int per_sm = 0, coop = 0;
    if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess || !coop) return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, select_coop<kMode>, kThreads, 0) != cudaSuccess)
      return 0;
    c = per_sm * sm_count();
    cap[dev].store(c, std::memory_order_relaxed);
  }
  return c;
}

// Runs the cooperative path when it applies; returns -1 when it does not.
template <int kMode>
int try_coop(const CoopArgs& ca, int64_t N, void* ws, size_t ws_bytes, int32_t* idx, int32_t* count,
             cudaStream_t st) {
  const int64_t G = coop_blocks(N);
  if (G > kCoopMaxBlocks || G > coop_capacity<kMode>() || ws_bytes < coop_bytes(N, kMode)) return -1;
  int err;
  unsigned int* status = device_status(&err);
  if (!status) return err;
  if (int e = cuda_status(cudaMemsetAsync(ws, 0, kCoopZeroWords * 4, st), "selection: clear barrier")) return e;
  CoopArgs a = ca;
  int64_t n = N;
  unsigned int* w = static_cast<unsigned int*>(ws);
  void* args[] = {&a, &n, &w, &idx, &count, &status};
  cudaError_t e = cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(select_coop<kMode>),
                                              dim3(static_cast<unsigned int>(G)), dim3(kThreads), args, 0, st);
  return cuda_status(e, "selection: cooperative launch");
}

// ---- host helpers ------------------------------------------------------------------
struct WsView {
  SelHdr* hdr;
  unsigned int* cnt;
  unsigned int* off;
};

inline int ncols_for(int op, int K) {
  if (op == TPS_OP_SELECT) return 2;
  if (op == TPS_OP_GROUP) return K > 1 ? K - 1 : 1;
  return 1;
}

// Minimum workspace: what the multi-launch path needs.
size_t ws_min_bytes(int op, int64_t N, int K) {
  const int64_t nb = n_blocks(N > 0 ? N : 1);
  return kHdrBytes + 2 * static_cast<size_t>(ncols_for(op, K)) * nb * sizeof(unsigned int);
}

// Recommended workspace: also enough for the single-launch cooperative path.
size_t ws_bytes_for(int op, int64_t N, int K) {
  const size_t classic = ws_min_bytes(op, N, K);
  size_t coop = 0;
  if (op != TPS_OP_GROUP && coop_blocks(N > 0 ? N : 1) <= kCoopMaxBlocks)
    coop = coop_bytes(N > 0 ? N : 1, op == TPS_OP_SELECT ? kCoopTopk : kCoopSched);
  return classic > coop ? classic : coop;
}

int check_ws(void* ws, size_t bytes, int op, int64_t N, int K, WsView* v, const char* who) {
  if (!ws) return fail(TPS_ERR_WORKSPACE, "%s: workspace is null", who);
  if (!aligned16(ws)) return fail(TPS_ERR_ALIGN, "%s: workspace must be 16-byte aligned", who);
  const size_t need = ws_min_bytes(op, N, K);
  if (bytes < need)
    return fail(TPS_ERR_WORKSPACE, "%s: workspace %zu bytes < required %zu", who, bytes, need);
  const int64_t nb = n_blocks(N);
  v->hdr = static_cast<SelHdr*>(ws);
  v->cnt = reinterpret_cast<unsigned int*>(static_cast<char*>(ws) + kHdrBytes);
  v->off = v->cnt + static_cast<size_t>(ncols_for(op, K)) * nb;
  return TPS_OK;
}

unsigned int radix_grid(int64_t N) {
  int64_t g = (N + 4 * kThreads - 1) / (4 * kThreads);
  const int64_t cap = static_cast<int64_t>(sm_count()) * 4;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<unsigned int>(g);
}

int run_radix(const float* s, int64_t N, SelHdr* h, int nbound, const Cuts& cuts, cudaStream_t st) {
  sel_init<<<1, kThreads, 0, st>>>(h, nbound, cuts);
  const unsigned int g = radix_grid(N);
  for (int shift = 24; shift >= 0; shift -= 8) radix_pass<<<g, kThreads, 0, st>>>(s, N, h, nbound, shift);
  return launch_status("radix select");
}

template <class Cls>
int run_compact(const Cls& cls, int64_t N, const WsView& v, int ncol, int32_t* idx, int32_t* count,
                cudaStream_t st, bool need_init) {
  if (need_init) sel_init<<<1, kThreads, 0, st>>>(v.hdr, 0, Cuts{});
  const unsigned int nb = static_cast<unsigned int>(n_blocks(N));
  compact_count<Cls><<<nb, kThreads, 0, st>>>(cls, N, v.hdr, v.cnt, v.off, ncol, count);
  compact_write<Cls><<<nb, kThreads, 0, st>>>(cls, N, v.hdr, v.off, ncol, idx);
  return launch_status("compaction");
}

}  // namespace
}  // namespace tps

extern "C" size_t tps_workspace_size(int op, int64_t N, int K) {
  if (op != TPS_OP_SELECT && op != TPS_OP_GROUP && op != TPS_OP_SCHEDULE) return 0;
  if (N < 0) return 0;
  return tps::ws_bytes_for(op, N, K);
}

extern "C" size_t tps_workspace_min_size(int op, int64_t N, int K) {
  if (op != TPS_OP_SELECT && op != TPS_OP_GROUP && op != TPS_OP_SCHEDULE) return 0;
  if (N < 0) return 0;
  return tps::ws_min_bytes(op, N, K);
}

extern "C" int lipar_select(const float* score, int64_t N, int mode, float tau, int64_t k,
                            int32_t* idx, int32_t* count, void* ws, size_t ws_bytes,
                            tps_stream stream) {
  TPS_TRACE("lipar_select");
  using namespace tps;
  if (mode != TPS_SELECT_THRESHOLD && mode != TPS_SELECT_TOPK)
    return fail(TPS_ERR_INVALID_ARG, "lipar_select: mode %d is not 0 (threshold) or 1 (top-k)", mode);
  if (!count) return fail(TPS_ERR_INVALID_ARG, "lipar_select: count must be non-null");
  if (N < 0 || N >= (INT64_C(1) << 31)) return fail(TPS_ERR_SHAPE, "lipar_select: N=%lld out of [0, 2^31)", (long long)N);
  if (mode == TPS_SELECT_TOPK && (k < 0 || k > N))
    return fail(TPS_ERR_INVALID_ARG, "lipar_select: k=%lld not in [0, N=%lld]", (long long)k, (long long)N);
  if (N > 0 && (!score || !idx)) return fail(TPS_ERR_INVALID_ARG, "lipar_select: score and idx must be non-null");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (N == 0 || (mode == TPS_SELECT_TOPK && k == 0)) {
    if (int e = cuda_status(cudaMemsetAsync(count, 0, sizeof(int32_t), st), "lipar_select: clear count")) return e;
    return ok();
  }
  WsView v;
  if (int e = check_ws(ws, ws_bytes, TPS_OP_SELECT, N, 0, &v, "lipar_select")) return e;
  int e;
  {
    CoopArgs ca{score, tau, nullptr, 0u, 0, static_cast<unsigned int>(k)};
    e = mode == TPS_SELECT_THRESHOLD ? try_coop<kCoopThresh>(ca, N, ws, ws_bytes, idx, count, st)
                                     : try_coop<kCoopTopk>(ca, N, ws, ws_bytes, idx, count, st);
    if (e >= 0) return e ? e : ok();
  }
  if (mode == TPS_SELECT_THRESHOLD) {
    e = run_compact(ThreshCls{score, tau}, N, v, 1, idx, count, st, true);
  } else {
    Cuts c{};
    c.k[0] = static_cast<unsigned int>(k);
    if ((e = run_radix(score, N, v.hdr, 1, c, st))) return e;
    e = run_compact(TopkCls{score}, N, v, 2, idx, count, st, false);
  }
  return e ? e : ok();
}

extern "C" int lipar_group(const float* score, int64_t N, int K, int8_t* group, void* ws,
                           size_t ws_bytes, tps_stream stream) {
  TPS_TRACE("lipar_group");
  using namespace tps;
  if (!score || !group) return fail(TPS_ERR_INVALID_ARG, "lipar_group: score and group must be non-null");
  if (N < 1 || N >= (INT64_C(1) << 31)) return fail(TPS_ERR_SHAPE, "lipar_group: N=%lld out of [1, 2^31)", (long long)N);
  if (K < 1 || K > kMaxBound + 1 || K > N)
    return fail(TPS_ERR_INVALID_ARG, "lipar_group: K=%d must be in [1, 8] and <= N", K);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (K == 1) {
    if (int e = cuda_status(cudaMemsetAsync(group, 0, static_cast<size_t>(N), st), "lipar_group: fill")) return e;
    return ok();
  }
  WsView v;
  if (int e = check_ws(ws, ws_bytes, TPS_OP_GROUP, N, K, &v, "lipar_group")) return e;
  const int nbound = K - 1;
  Cuts c{};
  const int64_t size = N / K;
  for (int b = 0; b < nbound; ++b) c.k[b] = static_cast<unsigned int>((b + 1) * size);
  if (int e = run_radix(score, N, v.hdr, nbound, c, st)) return e;
  const unsigned int nb = static_cast<unsigned int>(n_blocks(N));
  group_count<<<nb, kThreads, 0, st>>>(score, N, v.hdr, nbound, v.cnt, v.off);
  group_write<<<nb, kThreads, 0, st>>>(score, N, v.hdr, nbound, v.off, group);
  if (int e = launch_status("lipar_group")) return e;
  return ok();
}

extern "C" int lipar_schedule(const int8_t* group, int64_t N, int K, const int32_t* budgets, int T,
                              int step, int m, int32_t* idx, int32_t* count, void* ws,
                              size_t ws_bytes, tps_stream stream) {
  TPS_TRACE("lipar_schedule");
  using namespace tps;
  if (!count || !budgets) return fail(TPS_ERR_INVALID_ARG, "lipar_schedule: count and budgets must be non-null");
  if (N < 0 || N >= (INT64_C(1) << 31)) return fail(TPS_ERR_SHAPE, "lipar_schedule: N=%lld out of [0, 2^31)", (long long)N);
  if (K < 1 || K > 8) return fail(TPS_ERR_INVALID_ARG, "lipar_schedule: K=%d must be in [1, 8]", K);
  if (T < 1 || step < 0 || step >= T || m < 0)
    return fail(TPS_ERR_INVALID_ARG, "lipar_schedule: need T >= 1, 0 <= step < T, m >= 0");
  unsigned int act = 0;
  for (int g = 0; g < K; ++g) {
    const int s = budgets[g];
    if (s < 1 || s > T || T % s)
      return fail(TPS_ERR_INVALID_ARG, "lipar_schedule: budget[%d]=%d must divide T=%d", g, s, T);
    const bool full = step < m || step >= T - m;
    if (full || step % (T / s) == 0) act |= 1u << g;
  }
  if (N > 0 && (!group || !idx)) return fail(TPS_ERR_INVALID_ARG, "lipar_schedule: group and idx must be non-null");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (N == 0) {
    if (int e = cuda_status(cudaMemsetAsync(count, 0, sizeof(int32_t), st), "lipar_schedule: clear count")) return e;
    return ok();
  }
  WsView v;
  if (int e = check_ws(ws, ws_bytes, TPS_OP_SCHEDULE, N, K, &v, "lipar_schedule")) return e;
  {
    CoopArgs ca{nullptr, 0.f, group, act, K, 0u};
    const int e = try_coop<kCoopSched>(ca, N, ws, ws_bytes, idx, count, st);
    if (e >= 0) return e ? e : ok();
  }
  if (int e = run_compact(SchedCls{group, act, K}, N, v, 1, idx, count, st, true)) return e;
  return ok();
}

// ---- allocation-free variant of lipar_select ------------------------------------------
// Some callers cannot hand the library a workspace: a C host that runs the
// step inside a fixed device-memory plan (every buffer owned by the model
// runtime, none spare), or a latency-critical denoising loop that must not call
// cudaMalloc, which synchronises the device. For them the selection scratch
// lives in a file-scope device array sized for at most kStaticMaxN tokens.
// Every GPU that loads the library holds this array (about 73 KB) until the
// process exits.
namespace tps {
namespace {
constexpr int64_t kStaticMaxN = INT64_C(1) << 22;   // 4,194,304 tokens
constexpr size_t kStaticBytes =
    kHdrBytes + 2 * 2 * static_cast<size_t>((kStaticMaxN + kTile - 1) / kTile) * sizeof(unsigned int);
static __device__ __align__(256) unsigned char g_select_scratch[kStaticBytes];

// Device address of g_select_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// the device current. Devices 0..kCachedDevices-1 cache it after the first
// call; a device with a higher index looks it up on every call (still no
// allocation). The cache is not told about a context that is torn down and
// recreated (cudaDeviceReset): such a caller must not use this entry point
// after the reset.
constexpr int kCachedDevices = 64;
int static_scratch(void** out) {
  static void* ptrs[kCachedDevices] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e, "lipar_select_static: cudaGetDevice");
  const bool cacheable = dev >= 0 && dev < kCachedDevices;
  std::lock_guard<std::mutex> lk(mu);
  if (!cacheable || !ptrs[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_select_scratch);
    if (e != cudaSuccess) return cuda_status(e, "lipar_select_static: cudaGetSymbolAddress");
    if (!cacheable) {
      *out = p;
      return TPS_OK;
    }
    ptrs[dev] = p;
  }
  *out = ptrs[dev];
  return TPS_OK;
}
}  // namespace
}  // namespace tps

extern "C" int lipar_select_static(const float* score, int64_t N, int mode, float tau, int64_t k,
                                   int32_t* idx, int32_t* count, tps_stream stream) {
  TPS_TRACE("lipar_select_static");
  using namespace tps;
  if (N > kStaticMaxN)
    return fail(TPS_ERR_SHAPE, "lipar_select_static: N=%lld exceeds the static scratch limit of %lld tokens "
                "(use lipar_select with a caller-provided workspace)", (long long)N, (long long)kStaticMaxN);
  void* ws = nullptr;
  if (int e = static_scratch(&ws)) return e;
  return lipar_select(score, N, mode, tau, k, idx, count, ws, kStaticBytes, stream);
}
