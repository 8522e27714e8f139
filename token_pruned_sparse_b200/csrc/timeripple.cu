// timeripple_score: Timeripple's per-axis similarity check of Q / K tokens.
//
// [TR] "Timeripple: Accelerating vDiTs by Understanding the Spatio-Temporal
// Correlations in Latent Space", Metodologia 2: for every token and head three
// independent checks run along t, x and y; each compares the token with its
// neighbour on that axis through a standard error over a window of channels,
// and the token is reusable when any check falls below its threshold (OR).
// Metodologia 3: the thresholds rise linearly over steps 11-21.
//
// HBM-bound design. A CTA owns a 16 x 8 tile of latent positions for one head
// and sweeps a run of frames. Per frame one TMA box of (TX+1) x (TY+1) tokens
// (the tile plus its left column and top row, zero-filled outside the grid)
// lands in shared memory with a 128-byte swizzle, double-buffered on two
// mbarriers, so the next frame streams in while this one is checked. The x and
// y neighbours come from the box; the t neighbour is the thread's own token of
// the previous frame, kept in registers. Every element is read from HBM once
// (halos come from L2) and each (token, head) writes one byte.
//
// Threads: d = 128 runs two channel halves of 64 in separate warp groups (so
// every branch on the channel windows is warp-uniform); the halves' partial sums
// meet in shared memory. d = 64 runs one half. When the windows are the
// rotary-group windows (the default split of d into t, x, y groups), each
// chunk's channel masks are compile-time constants: chunks outside a window
// emit no code and full chunks take the unmasked path. Other windows read their
// masks at run time.
#include "trace.cuh"
#include "tc_ptx.cuh"
#include "tma_host.cuh"

namespace tps {
namespace {

using namespace tc;

constexpr int kTX = 16, kTY = 8;                    // tile of latent positions
constexpr int kBoxCols = kTX + 1, kBoxRows = kTY + 1;
constexpr int kBoxBytes = kBoxCols * kBoxRows * 128;  // 64 bf16 channels per token
constexpr int kBoxStride = (kBoxBytes + 1023) / 1024 * 1024;  // swizzle atoms want 1 KB alignment
constexpr int kTile = kTX * kTY;                    // threads per channel half

template <int D>
struct Lay {
  static constexpr int kHalves = D / 64;
  static constexpr int kThreads = kTile * kHalves;
  static constexpr int kSlot = kBoxStride * kHalves;
  static constexpr int kRed = 2 * kSlot;            // float [2][3][kTile]: half 1's partial sums
  static constexpr int kBar = kRed + (kHalves == 2 ? 2 * 3 * kTile * 4 : 0);
  static constexpr int kBytes = kBar + 64;          // 2 mbarriers + abort flag
  static constexpr int kAlloc = kBytes + 1024;      // slack for aligning the base
};

struct TrParams {
  int F, Hs, Ws, H;
  int tiles_x, tiles;       // tiles per frame
  int chunk;                // frames per work item
  int start[3], len[3];
  float inv_len[3];
  float theta[3];
  int fixed_windows;        // 1: the windows are the rotary-group windows of d (compile-time masks)
  int64_t N;
  uint8_t* reuse;
  float* delta;
  unsigned int* status;
};

__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            int c4, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5, %6}], "
      "[%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar)
      : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}

// Box row r under the 128-byte swizzle, with the row's swizzle key folded into
// its address: the row starts on a 128-byte boundary (box is 1 KB aligned), so
// its 16-byte chunk j sits at row_key(box, r) ^ (j << 4).
__device__ __forceinline__ uint32_t row_key(uint32_t box, int r) {
  return (box + static_cast<uint32_t>(r) * 128u) | (static_cast<uint32_t>(r & 7) << 4);
}

__device__ __forceinline__ void unpack(const uint4& w, float2 (&f)[4]) {
  f[0] = make_float2(bf16lo(w.x), bf16hi(w.x));
  f[1] = make_float2(bf16lo(w.y), bf16hi(w.y));
  f[2] = make_float2(bf16lo(w.z), bf16hi(w.z));
  f[3] = make_float2(bf16lo(w.w), bf16hi(w.w));
}

// (n - c) for the two bf16 channels packed in w against their fp32 centre values:
// the mixed-precision subtraction takes the bf16 operand directly (widening is
// exact), one rounding, the same value as -(c - n).
__device__ __forceinline__ float2 sub_bf16x2_f32(uint32_t w, float2 c) {
  float2 r;
  asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %2;\n sub.rn.f32.bf16 %0, lo, %3;\n sub.rn.f32.bf16 %1, hi, %4;\n}"
      : "=f"(r.x), "=f"(r.y)
      : "r"(w), "f"(c.x), "f"(c.y));
  return r;
}

// s += sum over the chunk's channels in mask m (bit e = channel e) of (n_e - c_e)^2,
// two channels per packed square-and-add and two independent accumulators. The
// neighbour n stays packed as bf16 pairs (nw); only the centre c is widened.
__device__ __forceinline__ void sq_acc(float2 (&s)[2], const float2 (&c)[4], const uint4& nw, uint32_t m) {
  const uint32_t w[4] = {nw.x, nw.y, nw.z, nw.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float2 d = sub_bf16x2_f32(w[q], c[q]);
    if (m != 0xffu) {
      d.x = (m >> (2 * q)) & 1u ? d.x : 0.f;
      d.y = (m >> (2 * q + 1)) & 1u ? d.y : 0.f;
    }
    s[q & 1] = __ffma2_rn(d, d, s[q & 1]);
  }
}

// Bits [lo, hi) of a 64-bit mask, clamped to [0, 64].
__device__ __forceinline__ uint64_t bit_range(int lo, int hi) {
  lo = lo < 0 ? 0 : (lo > 64 ? 64 : lo);
  hi = hi < 0 ? 0 : (hi > 64 ? 64 : hi);
  if (hi <= lo) return 0;
  const uint64_t upto_hi = hi == 64 ? ~0ull : ((1ull << hi) - 1);
  return upto_hi & ~((1ull << lo) - 1);
}

// Channels 64*half .. 64*half+63 that fall in the cyclic window [s, s+len) mod d.
__device__ __forceinline__ uint64_t window_mask(int s, int len, int d, int half) {
  const int b = 64 * half;
  uint64_t m = bit_range(s - b, (s + len < d ? s + len : d) - b);
  if (s + len > d) m |= bit_range(-b, s + len - d - b);
  return m;
}

// The configured windows (rotary groups [t | x | y] of sizes d - 4*(d/6), 2*(d/6),
// 2*(d/6); each check uses the groups its axis does not rotate), as (start, len)
// per axis. When a call passes exactly these, the chunk masks below are
// compile-time constants and the per-chunk branches on them disappear.
__host__ __device__ constexpr int fixed_window(int d, int a, int which) {
  return a == 0 ? (which == 0 ? d - 4 * (d / 6) : 4 * (d / 6))
       : a == 1 ? (which == 0 ? d - 2 * (d / 6) : d - 2 * (d / 6))
                : (which == 0 ? 0 : d - 2 * (d / 6));
}

// 8-bit mask of chunk j (channels c0 .. c0+7) in the cyclic window [s, s+len) mod d.
__host__ __device__ constexpr uint32_t chunk_bits(int s, int len, int d, int c0) {
  uint32_t m = 0;
  for (int e = 0; e < 8; ++e) m |= (((c0 + e - s) % d + d) % d < len ? 1u : 0u) << e;
  return m;
}

template <int D, int HALF, int J, int A>
__device__ __forceinline__ constexpr uint32_t fixed_bits() {
  return chunk_bits(fixed_window(D, A, 0), fixed_window(D, A, 1), D, 64 * HALF + 8 * J);
}

// The checks of one frame for this thread's token and 64 channels: chunk j+1's
// three rows are loaded while chunk j is checked. kFixed: compile-time windows.
template <int D, int HALF, bool kFixed>
__device__ __forceinline__ void check_frame(uint32_t box, int rc, bool has_t, const uint32_t (&pin)[32],
                                            uint32_t (&pout)[32], float2 (&at)[2],
                                            float2 (&ax)[2], float2 (&ay)[2], const uint32_t (&wlo)[3],
                                            const uint32_t (&whi)[3]) {
  const uint32_t kc = row_key(box, rc), kl = row_key(box, rc - 1), ku = row_key(box, rc - kBoxCols);
  uint4 ncw = lds128(kc), nlw = lds128(kl), nuw = lds128(ku);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint4 cw = ncw, lw = nlw, uw = nuw;
    if (j < 7) {
      ncw = lds128(kc ^ static_cast<uint32_t>((j + 1) << 4));
      nlw = lds128(kl ^ static_cast<uint32_t>((j + 1) << 4));
      nuw = lds128(ku ^ static_cast<uint32_t>((j + 1) << 4));
    }
    float2 c[4];
    unpack(cw, c);
    uint32_t mt, mx, my;
    if constexpr (kFixed) {
      // j is a compile-time constant after unrolling
      constexpr uint32_t f0[8] = {fixed_bits<D, HALF, 0, 0>(), fixed_bits<D, HALF, 1, 0>(), fixed_bits<D, HALF, 2, 0>(),
                                  fixed_bits<D, HALF, 3, 0>(), fixed_bits<D, HALF, 4, 0>(), fixed_bits<D, HALF, 5, 0>(),
                                  fixed_bits<D, HALF, 6, 0>(), fixed_bits<D, HALF, 7, 0>()};
      constexpr uint32_t f1[8] = {fixed_bits<D, HALF, 0, 1>(), fixed_bits<D, HALF, 1, 1>(), fixed_bits<D, HALF, 2, 1>(),
                                  fixed_bits<D, HALF, 3, 1>(), fixed_bits<D, HALF, 4, 1>(), fixed_bits<D, HALF, 5, 1>(),
                                  fixed_bits<D, HALF, 6, 1>(), fixed_bits<D, HALF, 7, 1>()};
      constexpr uint32_t f2[8] = {fixed_bits<D, HALF, 0, 2>(), fixed_bits<D, HALF, 1, 2>(), fixed_bits<D, HALF, 2, 2>(),
                                  fixed_bits<D, HALF, 3, 2>(), fixed_bits<D, HALF, 4, 2>(), fixed_bits<D, HALF, 5, 2>(),
                                  fixed_bits<D, HALF, 6, 2>(), fixed_bits<D, HALF, 7, 2>()};
      mt = f0[j], mx = f1[j], my = f2[j];
    } else {
      mt = j < 4 ? (wlo[0] >> (8 * j)) & 0xffu : (whi[0] >> (8 * (j - 4))) & 0xffu;
      mx = j < 4 ? (wlo[1] >> (8 * j)) & 0xffu : (whi[1] >> (8 * (j - 4))) & 0xffu;
      my = j < 4 ? (wlo[2] >> (8 * j)) & 0xffu : (whi[2] >> (8 * (j - 4))) & 0xffu;
    }
    if (has_t && mt) sq_acc(at, c, make_uint4(pin[4 * j], pin[4 * j + 1], pin[4 * j + 2], pin[4 * j + 3]), mt);
    if (mx) sq_acc(ax, c, lw, mx);
    if (my) sq_acc(ay, c, uw, my);
    pout[4 * j] = cw.x, pout[4 * j + 1] = cw.y, pout[4 * j + 2] = cw.z, pout[4 * j + 3] = cw.w;
  }
}

template <int D>
__global__ void __launch_bounds__(Lay<D>::kThreads, 2) tr_kernel(const __grid_constant__ CUtensorMap tm, TrParams p) {
  using L = Lay<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  const uint32_t bar0 = sbase + L::kBar, bar1 = bar0 + 8;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kBar + 16);
  float* red = reinterpret_cast<float*>(sm + L::kRed);

  const int tid = threadIdx.x;
  const int half = tid / kTile;                      // warp-uniform
  const int t = tid % kTile;
  const int ty = t / kTX, tx = t % kTX;

  int item = blockIdx.x;                             // head fastest, then tile, then frame run
  const int h = item % p.H;
  item /= p.H;
  const int tile = item % p.tiles;
  const int run = item / p.tiles;
  const int y0 = (tile / p.tiles_x) * kTY, x0 = (tile % p.tiles_x) * kTX;
  const int f0 = run * p.chunk;
  const int f1 = min(f0 + p.chunk, p.F);
  const int gy = y0 + ty, gx = x0 + tx;
  const bool inb = gy < p.Hs && gx < p.Ws;
  const int fstart = f0 > 0 ? f0 - 1 : 0;            // a run after the first primes with frame f0-1
  const int nload = f1 - fstart;

  if (tid == 0) {
    mbar_init(bar0, 1);
    mbar_init(bar1, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm);
  }
  __syncthreads();

  auto issue = [&](int k) {
    const uint32_t bar = (k & 1) ? bar1 : bar0;
    const uint32_t slot = sbase + static_cast<uint32_t>((k & 1) * L::kSlot);
    mbar_expect_tx(bar, static_cast<uint32_t>(L::kHalves * kBoxBytes));
#pragma unroll
    for (int hh = 0; hh < L::kHalves; ++hh)
      tma_load_5d(slot + hh * kBoxStride, &tm, 64 * hh, h, x0 - 1, y0 - 1, fstart + k, bar);
  };
  int issued = 0;
  if (tid == 0) {
    for (; issued < 2 && issued < nload; ++issued) issue(issued);
  }

  uint32_t wlo[3], whi[3];                           // window masks of this half's channels 0-31, 32-63
#pragma unroll
  for (int a = 0; a < 3; ++a) {
    const uint64_t wm = p.len[a] > 0 ? window_mask(p.start[a], p.len[a], D, half) : 0ull;
    wlo[a] = static_cast<uint32_t>(wm), whi[a] = static_cast<uint32_t>(wm >> 32);
  }
  const int rc = (ty + 1) * kBoxCols + (tx + 1);     // this token's box row; left = rc-1, up = rc-kBoxCols
  uint32_t prev[32];                                 // previous frame, this thread's 64 channels
#pragma unroll
  for (int i = 0; i < 32; ++i) prev[i] = 0;

  // one frame: checks against pin (the previous frame), this frame's centres into pout;
  // false when a wait gave up (the CTA leaves together)
  auto step = [&](int k, const uint32_t (&pin)[32], uint32_t (&pout)[32]) -> bool {
    const uint32_t bar = (k & 1) ? bar1 : bar0;
    // a wait that gives up sets the abort flag; the CTA leaves together after the barrier below
    mbar_wait(bar, static_cast<uint32_t>((k >> 1) & 1), abort_flag, p.status);
    const int f = fstart + k;
    const uint32_t box = sbase + static_cast<uint32_t>((k & 1) * L::kSlot + half * kBoxStride);
    const bool prime = f < f0;
    const float2 z2 = make_float2(0.f, 0.f);
    float2 at[2] = {z2, z2}, ax[2] = {z2, z2}, ay[2] = {z2, z2};
    if (prime) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint4 c = lds128(row_key(box, rc) ^ static_cast<uint32_t>(j << 4));
        pout[4 * j] = c.x, pout[4 * j + 1] = c.y, pout[4 * j + 2] = c.z, pout[4 * j + 3] = c.w;
      }
    } else {
      const bool has_t = f > 0;
      if (p.fixed_windows) {
        if (half == 0) check_frame<D, 0, true>(box, rc, has_t, pin, pout, at, ax, ay, wlo, whi);
        else check_frame<D, (L::kHalves > 1 ? 1 : 0), true>(box, rc, has_t, pin, pout, at, ax, ay, wlo, whi);
      } else {
        check_frame<D, 0, false>(box, rc, has_t, pin, pout, at, ax, ay, wlo, whi);
      }
    }
    float s[3] = {(at[0].x + at[1].x) + (at[0].y + at[1].y), (ax[0].x + ax[1].x) + (ax[0].y + ax[1].y),
                  (ay[0].x + ay[1].x) + (ay[0].y + ay[1].y)};
    float* r = red + (k & 1) * 3 * kTile;
    if (L::kHalves == 2 && half == 1 && !prime) r[t] = s[0], r[kTile + t] = s[1], r[2 * kTile + t] = s[2];
    __syncthreads();                                 // slot consumed, partial sums visible
    if (*abort_flag) return false;                   // same value in every thread: set before the barrier
    if (tid == 0 && issued < nload) {
      fence_proxy_async_smem();
      issue(issued++);
    }
    if (prime || half != 0 || !inb) return true;
    if (L::kHalves == 2) s[0] += r[t], s[1] += r[kTile + t], s[2] += r[2 * kTile + t];
    const bool has[3] = {f > 0, gx > 0, gy > 0};
    const int64_t n = (static_cast<int64_t>(f) * p.Hs + gy) * p.Ws + gx;
    unsigned int bits = 0;
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      const float dl = (has[a] && p.len[a] > 0) ? sqrtf(s[a] * p.inv_len[a]) : INFINITY;
      bits |= (dl < p.theta[a] ? 1u : 0u) << a;
      if (p.delta) p.delta[(static_cast<int64_t>(a) * p.N + n) * p.H + h] = dl;
    }
    p.reuse[n * p.H + h] = static_cast<uint8_t>(bits);
    return true;
  };
  // two frames per iteration with the previous-frame arrays swapping roles, so a frame's
  // centres land in their registers for the next frame without a copy
  uint32_t prev2[32];
  int k = 0;
  while (k < nload) {
    if (!step(k, prev, prev2)) break;
    if (++k >= nload) break;
    if (!step(k, prev2, prev)) break;
    ++k;
  }
  if (k < nload && tid == 0) {                       // gave up: let this CTA's copies land first
    for (int kk = k; kk < issued; ++kk) drain_wait((kk & 1) ? bar1 : bar0, static_cast<uint32_t>((kk >> 1) & 1));
  }
}

// score[n] = number of heads of token n whose reuse byte is 0.
__global__ void tr_count_kernel(const uint8_t* __restrict__ reuse, int64_t N, int H, bool words,
                                float* __restrict__ score) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; n < N; n += stride) {
    const uint8_t* row = reuse + n * H;
    int c = 0;
    if (words) {
      const uint32_t* w = reinterpret_cast<const uint32_t*>(row);
      for (int i = 0; i < H / 4; ++i) c += __popc(__vcmpeq4(__ldg(w + i), 0u)) >> 3;
    } else {
      for (int i = 0; i < H; ++i) c += __ldg(row + i) == 0;
    }
    score[n] = static_cast<float>(c);
  }
}

// (d, H, Ws, Hs, F) map of x, box (64, 1, TX+1, TY+1, 1), 128-byte swizzle.
int make_map5(EncodeTiledFn enc, CUtensorMap* m, const void* x, int64_t F, int64_t Hs, int64_t Ws, int H, int d) {
  const cuuint64_t row = static_cast<cuuint64_t>(H) * d * 2;
  cuuint64_t dims[5] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(Ws),
                        static_cast<cuuint64_t>(Hs), static_cast<cuuint64_t>(F)};
  cuuint64_t strides[4] = {static_cast<cuuint64_t>(d) * 2, row, row * Ws, row * Ws * Hs};
  cuuint32_t box[5] = {64, 1, kBoxCols, kBoxRows, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(x), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(TPS_ERR_CUDA, "timeripple_score: cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return TPS_OK;
}

// Frames per work item: the run length that minimises (waves of CTAs) x
// (frames loaded per CTA, counting the priming frame of every run but the first).
int choose_chunk(int F, int64_t items_per_run, int64_t resident) {
  int best = F;
  int64_t best_cost = INT64_MAX;
  for (int runs = 1; runs <= F && runs <= 16; ++runs) {
    const int len = (F + runs - 1) / runs;
    const int nr = (F + len - 1) / len;
    const int64_t waves = (items_per_run * nr + resident - 1) / resident;
    const int64_t cost = waves * (len + (nr > 1 ? 1 : 0));
    if (cost < best_cost) best_cost = cost, best = len;
  }
  return best;
}

template <int D>
int launch(const tps_bf16* x, int64_t F, int64_t Hs, int64_t Ws, int H, TrParams p, cudaStream_t st) {
  using L = Lay<D>;
  EncodeTiledFn enc;
  if (int e = tensor_map_encoder(&enc, "timeripple_score")) return e;
  CUtensorMap tm;
  if (int e = make_map5(enc, &tm, x, F, Hs, Ws, H, D)) return e;
  // resident CTAs per SM, per device; nonzero once the smem attribute is set on that device
  static std::atomic<int> occ[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return fail(TPS_ERR_CUDA, "timeripple_score: device index %d", dev);
  int oc = occ[dev].load(std::memory_order_acquire);
  if (!oc) {
    cudaError_t e = cudaFuncSetAttribute(tr_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return cuda_status(e, "timeripple_score: smem attribute");
    int b = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, tr_kernel<D>, L::kThreads, L::kAlloc);
    if (e != cudaSuccess) return cuda_status(e, "timeripple_score: occupancy");
    oc = b > 0 ? b : 1;
    occ[dev].store(oc, std::memory_order_release);
  }
  p.tiles_x = static_cast<int>((Ws + kTX - 1) / kTX);
  p.tiles = p.tiles_x * static_cast<int>((Hs + kTY - 1) / kTY);
  const int64_t per_run = static_cast<int64_t>(p.tiles) * H;
  p.chunk = choose_chunk(static_cast<int>(F), per_run, static_cast<int64_t>(oc) * sm_count());
  const int64_t runs = (F + p.chunk - 1) / p.chunk;
  const int64_t grid = per_run * runs;
  if (grid > 0x7fffffff) return fail(TPS_ERR_SHAPE, "timeripple_score: %lld work items", (long long)grid);
  tr_kernel<D><<<static_cast<unsigned int>(grid), L::kThreads, L::kAlloc, st>>>(tm, p);
  return launch_status("timeripple_score");
}

}  // namespace
}  // namespace tps

extern "C" int timeripple_score(const tps_bf16* x, int64_t F, int64_t Hs, int64_t Ws, int H, int d,
                                const int32_t* windows, const float* theta, uint8_t* reuse, float* delta,
                                float* score, tps_stream stream) {
  TPS_TRACE("timeripple_score");
  using namespace tps;
  if (!x || !windows || !theta || !reuse) return fail(TPS_ERR_INVALID_ARG, "timeripple_score: null pointer");
  if (d != 64 && d != 128) return fail(TPS_ERR_INVALID_ARG, "timeripple_score: d=%d must be 64 or 128", d);
  if (F < 1 || Hs < 1 || Ws < 1 || H < 1 || F >= (INT64_C(1) << 31) || Hs >= (INT64_C(1) << 31) ||
      Ws >= (INT64_C(1) << 31) || H > 65535)
    return fail(TPS_ERR_SHAPE, "timeripple_score: need F, Hs, Ws >= 1 (< 2^31) and 1 <= H <= 65535");
  const int64_t N = F * Hs * Ws;
  if (N / F / Hs != Ws || N >= (INT64_C(1) << 40) / (static_cast<int64_t>(H) * d))
    return fail(TPS_ERR_SHAPE, "timeripple_score: tensor too large");
  TrParams p{};
  for (int a = 0; a < 3; ++a) {
    const int s = windows[2 * a], len = windows[2 * a + 1];
    if (s < 0 || s >= d || len < 0 || len > d)
      return fail(TPS_ERR_INVALID_ARG, "timeripple_score: window %d = (%d, %d) outside [0, d)", a, s, len);
    if (theta[a] != theta[a]) return fail(TPS_ERR_INVALID_ARG, "timeripple_score: theta[%d] is NaN", a);
    p.start[a] = s, p.len[a] = len, p.theta[a] = theta[a];
    p.inv_len[a] = len > 0 ? 1.0f / static_cast<float>(len) : 0.0f;
  }
  if (!aligned16(x)) return fail(TPS_ERR_ALIGN, "timeripple_score: x must be 16-byte aligned");
  int err;
  unsigned int* st = device_status(&err);
  if (!st) return err;
  p.fixed_windows = 1;
  for (int a = 0; a < 3; ++a)
    if (p.start[a] != fixed_window(d, a, 0) || p.len[a] != fixed_window(d, a, 1)) p.fixed_windows = 0;
  p.F = static_cast<int>(F), p.Hs = static_cast<int>(Hs), p.Ws = static_cast<int>(Ws), p.H = H;
  p.N = N, p.reuse = reuse, p.delta = delta, p.status = st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (int e = (d == 128 ? launch<128>(x, F, Hs, Ws, H, p, s) : launch<64>(x, F, Hs, Ws, H, p, s))) return e;
  if (score) {
    int64_t blocks = (N + 255) / 256;
    const int64_t maxb = static_cast<int64_t>(sm_count()) * 8;
    if (blocks > maxb) blocks = maxb;
    const bool words = (H & 3) == 0 && (reinterpret_cast<uintptr_t>(reuse) & 3u) == 0;
    tr_count_kernel<<<static_cast<unsigned int>(blocks), 256, 0, s>>>(reuse, N, H, words, score);
    if (int e = launch_status("timeripple_score (token count)")) return e;
  }
  return ok();
}

extern "C" float timeripple_theta(int step, float theta_lo, float theta_hi, int i0, int i1) {
  if (step <= i0) return theta_lo;
  if (step >= i1) return theta_hi;
  return theta_lo + (theta_hi - theta_lo) * static_cast<float>(step - i0) / static_cast<float>(i1 - i0);
}
