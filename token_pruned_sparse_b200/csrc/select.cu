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

// ---- single-launch cooperative path (threshold, top-k, schedule, group) -------------
// For N up to 256 blocks of 256*kItems elements the whole selection runs as ONE
// cooperative launch (all blocks co-resident, guaranteed by the launch): each
// block keeps its keys in registers; the four radix passes and the final
// compaction (or, for groups, the tie ranking) are separated by grid barriers.
// A barrier is a counter in the workspace (zeroed before the launch) that
// thread 0 of every block increments and then polls; each poll loop is bounded
// by clock64 and, if it expires, sets the device status word (TPS_ERR_TIMEOUT)
// and the block leaves without writing results.
//
// With kV > 0 the launch also computes the scores (the fused front end,
// lipar_front): every block first scores its own tokens -- the relative L1
// change, with the same lane layout and summation order as lipar_score, so
// the scores are bit-identical -- into shared memory, and the selection reads
// them from there: the scores never make a round trip through global memory
// between the two stages.
constexpr int kCoopItems = 8;
constexpr int kCoopMaxBlocks = 256;
constexpr long long kGridWaitCycles = 2000000000LL; // ~1 s
constexpr int kCoopHdrWords = 64;                   // barrier counter + padding

enum CoopMode { kCoopThresh = 0, kCoopTopk = 1, kCoopSched = 2, kCoopGroup = 3 };

struct CoopArgs {
  const float* s;          // scores (kV == 0)
  float tau;
  const int8_t* g;         // groups (schedule)
  unsigned int act;
  int K;
  unsigned int k;          // top-k target (>= 1)
  int nbound;              // group: rank cuts (K - 1)
  unsigned int cuts[kMaxBound];
  int8_t* group;           // group: output
  const uint16_t* x;       // kV > 0: the tokens to score (as lipar_score)
  const uint16_t* xref;
  const uint16_t* xprev;
  int64_t HW;
  float* score_out;        // kV > 0: optional copy of the scores
};

inline int64_t coop_blocks(int64_t N, int items = kCoopItems) {
  return (N + kThreads * items - 1) / (kThreads * items);
}
// Workspace: header (barrier counter), the radix histograms (one 256-bin
// histogram per pass and cut, summed with atomics; zeroed with the header
// before the launch), then the per-block count columns.
__host__ __device__ inline int coop_zero_words(int mode, int nbound) {
  return kCoopHdrWords + (mode == kCoopGroup ? 4 * nbound * 256 : 4 * 256);
}
inline int coop_cols(int mode, int nbound) { return mode == kCoopGroup ? nbound : 2; }
inline size_t coop_bytes(int64_t G, int mode, int nbound) {
  return static_cast<size_t>(coop_zero_words(mode, nbound)) * 4 + static_cast<size_t>(G) * coop_cols(mode, nbound) * 4;
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

// Scores of this block's tokens into s_sc (fused front end). Eight lanes per
// token, 16-byte vectors, the same per-lane order and xor-shuffle reduction as
// score_kernel<8, kV, *>, hence the same fp32 result.
template <int kItems, int kV>
__device__ __forceinline__ void score_tile(const CoopArgs& a, int64_t N, float* s_sc) {
  constexpr int L = 8, kTokW = 32 / L, C = kV * 8;
  constexpr int kTileC = kThreads * kItems;
  constexpr int kSteps = kTileC / (kWarps * kTokW);
  constexpr int kG = 4;                               // token groups per lane in flight (8 measured no faster)
  static_assert(kSteps % kG == 0, "score steps");
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, sub = lane & (L - 1);
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kTileC;
  for (int s0 = 0; s0 < kSteps; s0 += kG) {
    const uint16_t* cur[kG];
    const uint16_t* ref[kG];
    int jj[kG];
    bool valid[kG];
#pragma unroll
    for (int q = 0; q < kG; ++q) {
      const int j = ((s0 + q) * kWarps + w) * kTokW + lane / L;
      const int64_t t = t0 + j;
      jj[q] = j;
      valid[q] = t < N;
      ref[q] = nullptr;
      cur[q] = a.x + (valid[q] ? t : 0) * C;
      if (valid[q]) {
        if (a.xref) ref[q] = a.xref + t * C;
        else if (t >= a.HW) ref[q] = a.x + (t - a.HW) * C;
        else if (a.xprev) ref[q] = a.xprev + t * C;
      }
    }
    float num[kG], den[kG];
#pragma unroll
    for (int q = 0; q < kG; ++q) num[q] = 0.f, den[q] = 0.f;
#pragma unroll
    for (int v = sub; v < kV; v += L) {
      uint4 ca[kG], cb[kG];
#pragma unroll
      for (int q = 0; q < kG; ++q)
        if (ref[q]) {
          ca[q] = ld16(cur[q] + v * 8);
          cb[q] = ld16(ref[q] + v * 8);
        }
#pragma unroll
      for (int q = 0; q < kG; ++q)
        if (ref[q]) {
          const uint32_t aw[4] = {ca[q].x, ca[q].y, ca[q].z, ca[q].w};
          const uint32_t bw[4] = {cb[q].x, cb[q].y, cb[q].z, cb[q].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float c0 = bf16lo(aw[i]), c1 = bf16hi(aw[i]);
            const float r0 = bf16lo(bw[i]), r1 = bf16hi(bw[i]);
            num[q] += fabsf(c0 - r0) + fabsf(c1 - r1);
            den[q] += fabsf(r0) + fabsf(r1);
          }
        }
    }
#pragma unroll
    for (int q = 0; q < kG; ++q) {
#pragma unroll
      for (int o = L / 2; o > 0; o >>= 1) {
        num[q] += __shfl_xor_sync(0xffffffffu, num[q], o);
        den[q] += __shfl_xor_sync(0xffffffffu, den[q], o);
      }
      if (valid[q] && sub == 0) {
        float s;
        if (!ref[q]) s = INFINITY;                  // frame 0 without a predecessor
        else if (den[q] > 0.f) s = num[q] / den[q];
        else s = num[q] > 0.f ? INFINITY : 0.f;
        s_sc[jj[q]] = s;
        if (a.score_out) a.score_out[t0 + jj[q]] = s;
      }
    }
  }
  __syncthreads();
}

// At least two blocks per SM must stay resident: the fused launch of
// N = 118,800 tokens spreads over 233 blocks.
template <int kMode, int kItems, int kV>
__global__ void __launch_bounds__(kThreads, 2) select_coop(CoopArgs a, int64_t N, unsigned int* ws,
                                                        int32_t* __restrict__ idx, int32_t* __restrict__ count,
                                                        unsigned int* status) {
  constexpr int kTileC = kThreads * kItems;
  constexpr int kCuts = kMode == kCoopGroup ? kMaxBound : 1;
  __shared__ unsigned int sh[kCuts][256];
  __shared__ float s_sc[kV > 0 ? kTileC : 1];
  __shared__ unsigned int s_pref[kCuts], s_krem[kCuts];
  __shared__ volatile int s_fail;
  __shared__ unsigned int s_sel[kWarps], s_tie[kWarps];
  __shared__ unsigned int s_eq[kCuts][kWarps];
  const unsigned int G = gridDim.x, b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int nbound = kMode == kCoopGroup ? a.nbound : 1;
  unsigned int* bar = ws;
  unsigned int* hist = ws + kCoopHdrWords;                       // [4][cuts][256]
  unsigned int* cnt = ws + coop_zero_words(kMode, nbound);       // [G][cols]
  if (tid == 0) s_fail = 0;
  if constexpr (kV > 0) score_tile<kItems, kV>(a, N, s_sc);
  const int64_t base = static_cast<int64_t>(b) * kTileC + w * (32 * kItems);
  uint32_t key[kItems];
  int cls[kItems];
#pragma unroll
  for (int it = 0; it < kItems; ++it) {
    const int64_t n = base + it * 32 + lane;
    key[it] = 0u;
    cls[it] = 0;
    if (n < N) {
      if (kMode == kCoopSched) {
        const int v = a.g[n];
        cls[it] = (v >= 0 && v < a.K && ((a.act >> v) & 1u)) ? 1 : 0;
      } else {
        const float sv = kV > 0 ? s_sc[w * (32 * kItems) + it * 32 + lane] : a.s[n];
        if (kMode == kCoopThresh) cls[it] = sv >= a.tau ? 1 : 0;
        else key[it] = score_key(sv);
      }
    }
  }
  unsigned int nbar = 0;
  unsigned int krem = 0;
  if (kMode == kCoopTopk || kMode == kCoopGroup) {
    // MSB-first radix select of every cut at once: four 8-bit digits
    if (tid < nbound) {
      s_pref[tid] = 0u;
      s_krem[tid] = kMode == kCoopTopk ? a.k : a.cuts[tid];
    }
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      const unsigned int himask = pass == 0 ? 0u : (0xffffffffu << (shift + 8));
      for (int c = 0; c < nbound; ++c) sh[c][tid] = 0u;
      __syncthreads();
#pragma unroll
      for (int it = 0; it < kItems; ++it) {
        const int64_t n = base + it * 32 + lane;
        if (n < N)
          for (int c = 0; c < nbound; ++c)
            if ((key[it] & himask) == s_pref[c]) atomicAdd(&sh[c][(key[it] >> shift) & 255u], 1u);
      }
      __syncthreads();
      for (int c = 0; c < nbound; ++c)
        if (sh[c][tid]) atomicAdd(&hist[(pass * nbound + c) * 256u + tid], sh[c][tid]);   // one global histogram per pass and cut
      if (!grid_sync(bar, ++nbar * G, status, &s_fail)) return;
      for (int c = 0; c < nbound; ++c) {
        const unsigned int need = s_krem[c], pre = s_pref[c];
        const int bin = 255 - tid;                                // descending buckets
        const unsigned int v = __ldcg(&hist[(pass * nbound + c) * 256u + bin]);
        unsigned int tot;
        const unsigned int incl = block_incl_scan(v, &tot);
        const unsigned int excl = incl - v;
        if (excl < need && incl >= need) {
          s_pref[c] = pre | (static_cast<unsigned int>(bin) << shift);
          s_krem[c] = need - excl;
        }
        __syncthreads();
      }
    }
    if (kMode == kCoopTopk) {
      const unsigned int prefix = s_pref[0];
      krem = s_krem[0];
#pragma unroll
      for (int it = 0; it < kItems; ++it) {
        const int64_t n = base + it * 32 + lane;
        cls[it] = n >= N ? 0 : (key[it] > prefix ? 1 : (key[it] == prefix ? 2 : 0));
      }
    }
  }
  const unsigned int lt = (1u << lane) - 1u;
  if constexpr (kMode == kCoopGroup) {
    // ---- group: rank of each token among the ties at every cut, in index order
    for (int c = 0; c < nbound; ++c) {
      const unsigned int ks = s_pref[c];
      unsigned int weq = 0;
#pragma unroll
      for (int it = 0; it < kItems; ++it) {
        const int64_t n = base + it * 32 + lane;
        weq += __popc(__ballot_sync(0xffffffffu, n < N && key[it] == ks));
      }
      if (lane == 0) s_eq[c][w] = weq;
    }
    __syncthreads();
    if (tid < nbound) {
      unsigned int t = 0;
      for (int i = 0; i < kWarps; ++i) t += s_eq[tid][i];
      cnt[b * nbound + tid] = t;
    }
    if (!grid_sync(bar, ++nbar * G, status, &s_fail)) return;
    int grp[kItems];
#pragma unroll
    for (int it = 0; it < kItems; ++it) grp[it] = 0;
    for (int c = 0; c < nbound; ++c) {
      unsigned int ps = 0;
      for (unsigned int g = tid; g < b; g += kThreads) ps += __ldcg(&cnt[g * nbound + c]);
      unsigned int eb = block_sum(ps);
      for (int i = 0; i < w; ++i) eb += s_eq[c][i];
      const unsigned int ks = s_pref[c], kr = s_krem[c];
#pragma unroll
      for (int it = 0; it < kItems; ++it) {
        const int64_t n = base + it * 32 + lane;
        const unsigned int m = __ballot_sync(0xffffffffu, n < N && key[it] == ks);
        const unsigned int r = eb + __popc(m & lt);
        const bool above = key[it] > ks || (key[it] == ks && r < kr);
        grp[it] += above ? 0 : 1;
        eb += __popc(m);
      }
    }
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
      const int64_t n = base + it * 32 + lane;
      if (n < N) a.group[n] = static_cast<int8_t>(grp[it]);
    }
    return;
  }
  // ---- compaction ------------------------------------------------------------------
  unsigned int msel[kItems], mtie[kItems];
  unsigned int wsel = 0, wtie = 0;
#pragma unroll
  for (int it = 0; it < kItems; ++it) {
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

// Max co-resident blocks of a cooperative kernel on the current device (cached).
template <int kMode, int kItems, int kV>
int coop_capacity() {
  static std::atomic<int> cap[64];   // per device; two threads may both compute it, to the same value
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int c = cap[dev].load(std::memory_order_relaxed);
  if (!c) {
    int per_sm = 0, coop = 0;
    if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess || !coop) return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, select_coop<kMode, kItems, kV>, kThreads, 0) !=
        cudaSuccess)
      return 0;
    c = per_sm * sm_count();
    cap[dev].store(c, std::memory_order_relaxed);
  }
  return c;
}

// Runs the cooperative path when it applies; returns -1 when it does not.
template <int kMode, int kItems = kCoopItems, int kV = 0>
int try_coop(const CoopArgs& ca, int64_t N, void* ws, size_t ws_bytes, int32_t* idx, int32_t* count,
             cudaStream_t st) {
  const int64_t G = coop_blocks(N, kItems);
  const int nbound = kMode == kCoopGroup ? ca.nbound : 1;
  if (G > kCoopMaxBlocks || G > coop_capacity<kMode, kItems, kV>() || ws_bytes < coop_bytes(G, kMode, nbound))
    return -1;
  int err;
  unsigned int* status = device_status(&err);
  if (!status) return err;
  if (int e = cuda_status(cudaMemsetAsync(ws, 0, static_cast<size_t>(coop_zero_words(kMode, nbound)) * 4, st),
                          "selection: clear barrier"))
    return e;
  CoopArgs a = ca;
  int64_t n = N;
  unsigned int* w = static_cast<unsigned int*>(ws);
  void* args[] = {&a, &n, &w, &idx, &count, &status};
  cudaError_t e = cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(select_coop<kMode, kItems, kV>),
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
  const int64_t G = coop_blocks(N > 0 ? N : 1);
  if (G <= kCoopMaxBlocks)
    coop = op == TPS_OP_GROUP ? coop_bytes(G, kCoopGroup, K > 1 ? K - 1 : 1)
                              : coop_bytes(G, op == TPS_OP_SELECT ? kCoopTopk : kCoopSched, 1);
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

namespace tps {
namespace {
// lipar_front: a score scratch (used only when the fused launch does not apply
// and the caller passes no score array), then the selection / group workspace.
size_t front_score_bytes(int64_t N) { return (static_cast<size_t>(N > 0 ? N : 1) * 4 + 255) / 256 * 256; }
size_t front_min_bytes(int64_t N, int K) {
  const size_t a = ws_min_bytes(TPS_OP_SELECT, N, 0), b = ws_min_bytes(TPS_OP_GROUP, N, K);
  return front_score_bytes(N) + (a > b ? a : b);
}
size_t front_bytes(int64_t N, int K) {
  size_t m = ws_bytes_for(TPS_OP_SELECT, N, 0);
  const size_t g = ws_bytes_for(TPS_OP_GROUP, N, K);
  m = m > g ? m : g;
  const size_t f1 = coop_bytes(kCoopMaxBlocks, kCoopTopk, 1);
  const size_t f2 = coop_bytes(kCoopMaxBlocks, kCoopGroup, K > 1 ? (K - 1 < kMaxBound ? K - 1 : kMaxBound) : 1);
  m = m > f1 ? m : f1;
  m = m > f2 ? m : f2;
  return front_score_bytes(N) + m;
}
}  // namespace
}  // namespace tps

extern "C" size_t tps_workspace_size(int op, int64_t N, int K) {
  if (N < 0) return 0;
  if (op == TPS_OP_FRONT) return tps::front_bytes(N, K);
  if (op != TPS_OP_SELECT && op != TPS_OP_GROUP && op != TPS_OP_SCHEDULE) return 0;
  return tps::ws_bytes_for(op, N, K);
}

extern "C" size_t tps_workspace_min_size(int op, int64_t N, int K) {
  if (N < 0) return 0;
  if (op == TPS_OP_FRONT) return tps::front_min_bytes(N, K);
  if (op != TPS_OP_SELECT && op != TPS_OP_GROUP && op != TPS_OP_SCHEDULE) return 0;
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
    CoopArgs ca{};
    ca.s = score;
    ca.tau = tau;
    ca.k = static_cast<unsigned int>(k);
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
  {
    CoopArgs ca{};
    ca.s = score;
    ca.nbound = nbound;
    for (int b = 0; b < nbound; ++b) ca.cuts[b] = c.k[b];
    ca.group = group;
    const int e = try_coop<kCoopGroup>(ca, N, ws, ws_bytes, nullptr, nullptr, st);
    if (e >= 0) return e ? e : ok();
  }
  if (int e = run_radix(score, N, v.hdr, nbound, c, st)) return e;
  const unsigned int nb = static_cast<unsigned int>(n_blocks(N));
  group_count<<<nb, kThreads, 0, st>>>(score, N, v.hdr, nbound, v.cnt, v.off);
  group_write<<<nb, kThreads, 0, st>>>(score, N, v.hdr, nbound, v.off, group);
  if (int e = launch_status("lipar_group")) return e;
  return ok();
}

// ---- fused front end: score + selection (or group split) in one launch -------------
namespace tps {
namespace {
template <int kMode, int kV>
int front_coop(const CoopArgs& ca, int64_t N, void* ws, size_t ws_bytes, int32_t* idx, int32_t* count,
               cudaStream_t st) {
  if (coop_blocks(N, 2) <= kCoopMaxBlocks) return try_coop<kMode, 2, kV>(ca, N, ws, ws_bytes, idx, count, st);
  return try_coop<kMode, kCoopItems, kV>(ca, N, ws, ws_bytes, idx, count, st);
}
template <int kV>
int front_dispatch(int mode, const CoopArgs& ca, int64_t N, void* ws, size_t ws_bytes, int32_t* idx,
                   int32_t* count, cudaStream_t st) {
  if (mode == TPS_FRONT_THRESHOLD) return front_coop<kCoopThresh, kV>(ca, N, ws, ws_bytes, idx, count, st);
  if (mode == TPS_FRONT_TOPK) return front_coop<kCoopTopk, kV>(ca, N, ws, ws_bytes, idx, count, st);
  return front_coop<kCoopGroup, kV>(ca, N, ws, ws_bytes, idx, count, st);
}
}  // namespace
}  // namespace tps

extern "C" int lipar_front(const tps_bf16* x, const tps_bf16* x_ref, const tps_bf16* x_prev_frame, int64_t F,
                           int64_t HW, int64_t C, int mode, float tau, int64_t k, int K, float* score,
                           int32_t* idx, int32_t* count, int8_t* group, void* ws, size_t ws_bytes,
                           tps_stream stream) {
  TPS_TRACE("lipar_front");
  using namespace tps;
  if (!x) return fail(TPS_ERR_INVALID_ARG, "lipar_front: x must be non-null");
  if (F < 1 || HW < 1 || F > (INT64_C(1) << 31) / HW)
    return fail(TPS_ERR_SHAPE, "lipar_front: need F, HW >= 1 and F*HW < 2^31");
  if (C < 8 || C > 4096 || C % 8) return fail(TPS_ERR_SHAPE, "lipar_front: C=%lld must be a multiple of 8 in [8, 4096]", (long long)C);
  if (x_ref && x_prev_frame) return fail(TPS_ERR_INVALID_ARG, "lipar_front: x_prev_frame is for inter-frame mode only");
  const int64_t N = F * HW;
  if (mode == TPS_FRONT_THRESHOLD || mode == TPS_FRONT_TOPK) {
    if (!idx || !count) return fail(TPS_ERR_INVALID_ARG, "lipar_front: idx and count must be non-null");
    if (mode == TPS_FRONT_TOPK && (k < 0 || k > N))
      return fail(TPS_ERR_INVALID_ARG, "lipar_front: k=%lld not in [0, N=%lld]", (long long)k, (long long)N);
  } else if (mode == TPS_FRONT_GROUP) {
    if (!group) return fail(TPS_ERR_INVALID_ARG, "lipar_front: group must be non-null");
    if (K < 1 || K > kMaxBound + 1 || K > N)
      return fail(TPS_ERR_INVALID_ARG, "lipar_front: K=%d must be in [1, 8] and <= N", K);
  } else {
    return fail(TPS_ERR_INVALID_ARG, "lipar_front: mode %d is not 0 (threshold), 1 (top-k) or 2 (group)", mode);
  }
  if (!aligned16(x) || (x_ref && !aligned16(x_ref)) || (x_prev_frame && !aligned16(x_prev_frame)))
    return fail(TPS_ERR_ALIGN, "lipar_front: bf16 inputs must be 16-byte aligned");
  if (!ws) return fail(TPS_ERR_WORKSPACE, "lipar_front: workspace is null");
  if (!aligned16(ws)) return fail(TPS_ERR_ALIGN, "lipar_front: workspace must be 16-byte aligned");
  if (ws_bytes < front_min_bytes(N, K))
    return fail(TPS_ERR_WORKSPACE, "lipar_front: workspace %zu bytes < required %zu", ws_bytes, front_min_bytes(N, K));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool trivial = (mode == TPS_FRONT_TOPK && k == 0) || (mode == TPS_FRONT_GROUP && K == 1);
  if ((C == 128 || C == 64) && !trivial) {
    CoopArgs ca{};
    ca.tau = tau;
    ca.k = static_cast<unsigned int>(k);
    ca.nbound = mode == TPS_FRONT_GROUP ? K - 1 : 1;
    for (int b = 0; b + 1 < K && b < kMaxBound; ++b) ca.cuts[b] = static_cast<unsigned int>((b + 1) * (N / K));
    ca.group = group;
    ca.x = x;
    ca.xref = x_ref;
    ca.xprev = x_prev_frame;
    ca.HW = HW;
    ca.score_out = score;
    const int e = C == 128 ? front_dispatch<16>(mode, ca, N, ws, ws_bytes, idx, count, st)
                           : front_dispatch<8>(mode, ca, N, ws, ws_bytes, idx, count, st);
    if (e >= 0) return e ? e : ok();
  }
  // the separate kernels, with the scores in the caller's array or the workspace
  float* sbuf = score ? score : static_cast<float*>(ws);
  void* ws2 = static_cast<char*>(ws) + front_score_bytes(N);
  const size_t ws2_bytes = ws_bytes - front_score_bytes(N);
  if (int e = lipar_score(x, x_ref, x_prev_frame, F, HW, C, sbuf, stream)) return e;
  if (mode == TPS_FRONT_GROUP) return lipar_group(sbuf, N, K, group, ws2, ws2_bytes, stream);
  return lipar_select(sbuf, N, mode == TPS_FRONT_TOPK ? TPS_SELECT_TOPK : TPS_SELECT_THRESHOLD, tau, k, idx, count,
                      ws2, ws2_bytes, stream);
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
    CoopArgs ca{};
    ca.g = group;
    ca.act = act;
    ca.K = K;
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
