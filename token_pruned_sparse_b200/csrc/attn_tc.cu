// pruned_attn: active queries attend all N cached keys, on the Blackwell
// tensor cores (tcgen05 + TMEM + TMA).
//
// [HSA] "Asignacion de Pasos Heterogenea", 2.2 (3)-(4): the active tokens'
// queries attend the full cached K/V (fresh rows for active tokens, stale but
// valid rows for skipped ones), so the attention costs O(|A_i| * N).
// Key-block sparsity ([SVOO] part 2, co-clustering -> block-sparse attention;
// [TR] skipping of reusable work): with a mask, a query attends only the
// 128-key blocks its ORIGINAL 128-token block keeps.
//
// Dense mode: one CTA = 256 compacted active queries of one head, as two
// 128-row tiles (t = 0, 1) that share every K/V tile. Block mode (a mask is
// given), d = 64: tile t of CTA x holds the active rows of original query block
// 2x + t (at most 128; the rest of the tile is padding) and streams only the
// key tiles that block keeps, so every loaded key tile is work for every row
// of its tile; the two tiles' loads interleave in one K ring and one V ring.
// Block mode, d = 128: attn_blkt_kernel below, with the products transposed
// (keys as the MMA's M, at most 64 active rows of one query block as its N).
// In the dense and the d = 64 block kernel the two tiles take turns on the tensor cores:
//   warps 0-3 / 4-7  softmax of tile 0 / tile 1: thread r owns query row r of
//              its tile (= TMEM lane r). Loads S from TMEM, online softmax in
//              the log2 domain, writes P (bf16) back over the first half of
//              its S columns. After the first tile it skips the row maximum:
//              P is formed against the running reference maximum, which is
//              exact for any reference (the final normalisation uses the same
//              one), and only when a tile's row sum exceeds 2^40 does the warp
//              reload S, take the maximum and rescale O in TMEM.
//   warp 8     TMA producer: Q (both tiles) once, then K and V tiles of 128
//              keys into two-stage rings, 128-byte swizzled. A K stage is
//              freed when the last S MMA reading it completes and a V stage
//              when the last P V MMA does, so the next K tile streams in about
//              one tile period earlier than a shared K/V stage would allow.
//              (Block mode: each stage has one reader, its own tile.)
//   warp 9     MMA issuer and TMEM owner. Per key tile j and tile t:
//              O_t += P_t(j) V_j (A operand read from TMEM), then
//              S_t(j+1) = Q_t K_{j+1}^T; completion via tcgen05.commit.
//   warps 10-11 idle: with warps 8-9 they form a producer warpgroup that gives
//              up registers (setmaxnreg) so that each softmax thread holds S and P
//              of a whole tile (232 registers) without spilling.
// While softmax t works on S_t(j+1), the tensor cores run the other tile's
// P V and Q K^T, so MMA and softmax overlap.
// TMEM: tile t owns columns [256t, 256t+128) for S/P and [256t+128, +D) for O.
// Every mbarrier wait is bounded: on expiry the CTA sets an abort flag and the
// device status word (TPS_ERR_TIMEOUT via tps_check), drains what it issued,
// frees TMEM and returns.
#include "trace.cuh"
#include "attn_common.cuh"
#include "tc_ptx.cuh"
#include "tma_host.cuh"

namespace tps {
namespace {

using namespace tc;

constexpr int kBM = 128;        // query rows per tile (MMA M)
constexpr int kQT = 2;          // query tiles per CTA
constexpr int kBN = 128;        // keys per tile (MMA N of S, K of PV)
constexpr int kStages = 2;      // K/V ring depth
constexpr int kSoftmaxThreads = kQT * kBM;
// + a fourth warpgroup (TMA warp, MMA warp, two idle warps) that hands registers to
// the two softmax warpgroups (setmaxnreg). 12 warps put 3 on each SM sub-partition,
// so the launch allots 16384 / (3 * 32) -> 168 registers per thread; the softmax
// warps then hold S and P of a whole tile without spilling.
constexpr int kThreads = kSoftmaxThreads + 128;
constexpr int kLaunchRegs = 168;
constexpr int kProducerRegs = 40;
constexpr int kSoftmaxRegs = 232;
static_assert(8 * kSoftmaxRegs + 4 * kProducerRegs <= 12 * kLaunchRegs, "register split exceeds the launch");
constexpr int kTmaWarp = kSoftmaxThreads / 32;
constexpr int kMmaWarp = kTmaWarp + 1;
constexpr int kTmemCols = 512;
constexpr int kSubBytes = 128 * 128;   // one [128 rows x 64 bf16] swizzled sub-tile
constexpr float kSumLimit = 1099511627776.f;   // 2^40: largest tile row sum kept without a new max

// kLists: key-block lists (block mode: one per tile); the dense kernel's list
// region holds the (m, l) pairs of a cluster merge instead.
template <int D, int kLists>
struct Layout {
  static constexpr int kSub = D / 64;                    // 64-wide sub-tiles per row of Q/K/V
  static constexpr int kQ = 0;                           // [tile][sub]
  static constexpr int kK = kQ + kQT * kSub * kSubBytes; // [stage][sub]
  static constexpr int kV = kK + kStages * kSub * kSubBytes;
  static constexpr int kList = kV + kStages * kSub * kSubBytes;   // uint16 kept key blocks, per tile
  static constexpr int kListMax = 4096;
  static constexpr int kBar = kList + kLists * kListMax * 2;   // mbarriers (Bars)
  static constexpr int kBytes = kBar + 256;
  static constexpr int kAlloc = kBytes + 1024;           // slack for 1024-byte alignment
};

struct Bars {  // mbarrier indices inside the barrier block (8 bytes each)
  static constexpr int q_full = 0;                     // + tile
  static constexpr int k_full = q_full + kQT;          // + stage
  static constexpr int v_full = k_full + kStages;      // + stage
  static constexpr int k_empty = v_full + kStages;     // + stage: freed by the last S MMA reading it
  static constexpr int v_empty = k_empty + kStages;    // + stage: freed by the last PV MMA reading it
  static constexpr int s_full = v_empty + kStages;     // + tile
  static constexpr int p_full = s_full + kQT;          // + tile
  static constexpr int pv_done = p_full + kQT;         // + tile
  static constexpr int drain = pv_done + kQT;          // last commit of the MMA thread
  static constexpr int count = drain + 1;
};
static_assert(Bars::count * 8 <= 256, "barrier block");

struct TcParams {
  AttnArgs a;
  float scale_log2;
  unsigned int* status;
  int nsplit;          // key-range splits (blockIdx.z); 1 = whole key range
  float* o_part;       // nsplit > 1, workspace merge: normalised partial outputs, fp32 [nsplit][cap][H][D]
  float* lse_part;     // nsplit > 1, workspace merge: partial log-sum-exp, fp32 [nsplit][cap][H]
  int cluster;         // > 1: the nsplit CTAs of a cluster merge their partials over distributed
                       // shared memory (no workspace); 1 otherwise
  int tile0;           // dense mode: first 256-row query tile of this launch (blockIdx.x + tile0)
};
constexpr int kMaxCluster = 4;

// CTA and cluster barriers; the non-aligned forms when warps reach them from
// different code (each warpgroup running its own copy of the kernel's tail).
template <bool kNonAligned>
__device__ __forceinline__ void cta_sync() {
  if constexpr (kNonAligned) asm volatile("barrier.sync 0;" ::: "memory");
  else __syncthreads();
}
template <bool kNonAligned>
__device__ __forceinline__ void cluster_sync() {
  if constexpr (kNonAligned)
    asm volatile("barrier.cluster.arrive.release;\nbarrier.cluster.wait.acquire;" ::: "memory");
  else cluster_sync_all();
}


template <int D, bool kClu>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, TcParams prm) {
  using L = Layout<D, 1>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_ntiles;
  __shared__ volatile int s_abort;

  const AttnArgs& p = prm.a;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  const int64_t rows = active_count(p.count, p.cap);
  const int64_t row0 = (static_cast<int64_t>(blockIdx.x) + prm.tile0) * (kQT * kBM);
  if (row0 >= rows) return;   // whole CTA exits before touching TMEM or barriers

  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - smem_u32(smem_raw));
  const uint32_t bar0 = sbase + L::kBar;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  const int nkt_all = static_cast<int>((p.N + kBN - 1) / kBN);   // key tiles = key blocks
  // split z of nsplit (dense mode only) covers key tiles [kt0, kt0 + nkt)
  const int kt0 = static_cast<int>((static_cast<int64_t>(nkt_all) * blockIdx.z) / prm.nsplit);
  const int nkt = static_cast<int>((static_cast<int64_t>(nkt_all) * (blockIdx.z + 1)) / prm.nsplit) - kt0;

  // ---- setup: barriers, TMEM, key-tile list ---------------------------------------------
  if (tid == 0) {
    s_abort = 0;
    for (int t = 0; t < kQT; ++t) {
      mbar_init(bar(Bars::q_full + t), 1);
      mbar_init(bar(Bars::s_full + t), 1);
      mbar_init(bar(Bars::p_full + t), kBM);
      mbar_init(bar(Bars::pv_done + t), 1);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(Bars::k_full + s), 1);
      mbar_init(bar(Bars::v_full + s), 1);
      mbar_init(bar(Bars::k_empty + s), 1);
      mbar_init(bar(Bars::v_empty + s), 1);
    }
    mbar_init(bar(Bars::drain), 1);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tmem_alloc<kTmemCols>(smem_u32(&s_tmem));
  if (warp == kTmaWarp && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (tid == 0) s_ntiles = nkt;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int ntiles = s_ntiles;
  const uint32_t tmem = s_tmem;
  auto tS = [&](int t) { return tmem + 256u * t; };          // S_t, later P_t (bf16 pairs)
  auto tO = [&](int t) { return tmem + 256u * t + 128u; };   // O_t accumulator
  auto tile_kb = [&](int j) -> int { return kt0 + j; };

  auto tma_role = [&]() {
    // ================================ TMA producer =====================================
    if (lane == 0) {
      int issued_k = 0, issued_v = 0;
      for (int t = 0; t < kQT; ++t) {
        mbar_expect_tx(bar(Bars::q_full + t), L::kSub * kSubBytes);
        for (int s = 0; s < L::kSub; ++s)
          tma_load_3d(sbase + L::kQ + (t * L::kSub + s) * kSubBytes, &tmQ, 64 * s, h,
                      static_cast<int>(row0 + t * kBM), bar(Bars::q_full + t));
      }
      // K and V stages are freed separately: a K stage as soon as the last S MMA
      // reading it completes (about one period before its PV stage), so the next
      // K tile streams in while the current P.V products still run.
      for (int j = 0; j < ntiles; ++j) {
        const int st = j % kStages;
        const uint32_t ph = ((j / kStages) - 1) & 1;
        const int key0 = tile_kb(j) * kBN;
        if (j >= kStages && !mbar_wait(bar(Bars::k_empty + st), ph, &s_abort, prm.status)) break;
        mbar_expect_tx(bar(Bars::k_full + st), L::kSub * kSubBytes);
        for (int s = 0; s < L::kSub; ++s)
          tma_load_3d(sbase + L::kK + (st * L::kSub + s) * kSubBytes, &tmK, 64 * s, h, key0, bar(Bars::k_full + st));
        issued_k = j + 1;
        if (j >= kStages && !mbar_wait(bar(Bars::v_empty + st), ph, &s_abort, prm.status)) break;
        mbar_expect_tx(bar(Bars::v_full + st), L::kSub * kSubBytes);
        for (int s = 0; s < L::kSub; ++s)
          tma_load_3d(sbase + L::kV + (st * L::kSub + s) * kSubBytes, &tmV, 64 * s, h, key0, bar(Bars::v_full + st));
        issued_v = j + 1;
      }
      // drain: every load issued above must land before the CTA may exit
      for (int t = 0; t < kQT; ++t) drain_wait(bar(Bars::q_full + t), 0);
      for (int j = issued_k > kStages ? issued_k - kStages : 0; j < issued_k; ++j)
        drain_wait(bar(Bars::k_full + j % kStages), (j / kStages) & 1);
      for (int j = issued_v > kStages ? issued_v - kStages : 0; j < issued_v; ++j)
        drain_wait(bar(Bars::v_full + j % kStages), (j / kStages) & 1);
    }
  };
  auto mma_role = [&]() {
    // ================================ MMA issuer =======================================
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16(kBM, kBN, false, false);  // Q K^T: both K-major
      constexpr uint32_t kIdescO = idesc_bf16(kBM, D, false, true);     // P V: V is MN-major
      auto issue_s = [&](int t, int j) {
        const int st = j % kStages;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kSubBytes + (kk & 3) * 32;   // 16 bf16 along d
          const uint64_t da = sdesc_sw128(sbase + L::kQ + t * L::kSub * kSubBytes + off, 16, 1024);
          const uint64_t db = sdesc_sw128(sbase + L::kK + st * L::kSub * kSubBytes + off, 16, 1024);
          mma_f16_ss(tS(t), da, db, kIdescS, kk > 0);
        }
        mma_commit(bar(Bars::s_full + t));
        if (t == kQT - 1) mma_commit(bar(Bars::k_empty + st));   // last reader of this K stage
      };
      bool ok = ntiles > 0;
      if (ok) ok = mbar_wait(bar(Bars::k_full), 0, &s_abort, prm.status);
      for (int t = 0; ok && t < kQT; ++t) {
        ok = mbar_wait(bar(Bars::q_full + t), 0, &s_abort, prm.status);
        tc_fence_after();
        if (ok) issue_s(t, 0);
      }
      for (int j = 0; ok && j < ntiles; ++j) {
        const int st = j % kStages;
        for (int t = 0; ok && t < kQT; ++t) {
          ok = mbar_wait(bar(Bars::p_full + t), j & 1, &s_abort, prm.status);
          if (ok && t == 0) ok = mbar_wait(bar(Bars::v_full + st), (j / kStages) & 1, &s_abort, prm.status);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            // B = V [128 keys x D], MN-major: 16 keys = 2 swizzle atoms of 8 rows;
            // LBO = next 64-wide d sub-tile, SBO = next 8 keys. A = P_t from TMEM,
            // 16 keys = 8 columns of bf16 pairs.
            const uint64_t db = sdesc_sw128(sbase + L::kV + st * L::kSub * kSubBytes + kk * 16 * 128, kSubBytes, 1024);
            mma_f16_ts(tO(t), tS(t) + 8 * kk, db, kIdescO, (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar(Bars::pv_done + t));
          if (t == kQT - 1) mma_commit(bar(Bars::v_empty + st));   // last reader of this V stage
          if (j + 1 < ntiles) {
            // S_t(j+1) overwrites the columns P_t(j) was read from: tcgen05.mma
            // operations of one thread execute in issue order.
            if (t == 0) {
              ok = mbar_wait(bar(Bars::k_full + (j + 1) % kStages), ((j + 1) / kStages) & 1, &s_abort, prm.status);
              tc_fence_after();
            }
            if (ok) issue_s(t, j + 1);
          }
        }
      }
      mma_commit(bar(Bars::drain));   // fires once every MMA issued above has completed
    }
  };
  auto softmax_role = [&]() {
    // ================================ softmax warps ====================================
    const int t = warp >> 2;                      // query tile of this warpgroup
    const int r = (warp & 3) * 32 + lane;         // row within the tile == TMEM lane
    const int64_t row = row0 + t * kBM + r;
    const bool valid = row < rows;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float sl2 = prm.scale_log2;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      // every wait result is made warp-uniform: tcgen05.ld/st are .sync.aligned
      if (!__all_sync(0xffffffffu, mbar_wait(bar(Bars::s_full + t), j & 1, &s_abort, prm.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int64_t key0 = static_cast<int64_t>(tile_kb(j)) * kBN;
      const int nvalid = static_cast<int>(p.N - key0 < kBN ? p.N - key0 : kBN);
      uint32_t sr[kBN];
      auto load_s = [&]() {
        tmem_ld128(tS(t) + lane_off, sr);
        if (nvalid < kBN) {
#pragma unroll
          for (int c = 0; c < kBN; ++c)
            if (c >= nvalid) sr[c] = __float_as_uint(-INFINITY);
        }
      };
      uint32_t pk[kBN / 2];
      // P = exp2(S * scale_log2 - base) as bf16 pairs into pk; returns the row sum of this tile
      auto exp_pass = [&](float base) -> float { return exp_row<kBN>(sr, sl2x2, base, pk); };
      load_s();
      // Fast path: keep the running reference max and skip the row max. Softmax is
      // exact for any reference; the tile's sum bounds every P, so P stays finite
      // and well inside bf16/fp32 range while the sum is at most kSumLimit.
      bool slow = j == 0;
      float lt = 0.f;
      if (!slow) {
        const float base = m_run == -INFINITY ? 0.f : m_run;
        lt = exp_pass(base);
        slow = __any_sync(0xffffffffu, !(lt <= kSumLimit));
        if (slow) load_s();                         // S is intact: P has not been stored yet
        else m_run = base;                          // a row with only masked keys so far now uses 0
      }
      if (slow) {
        float mx0 = __uint_as_float(sr[0]), mx1 = __uint_as_float(sr[1]);
        float mx2 = __uint_as_float(sr[2]), mx3 = __uint_as_float(sr[3]);
#pragma unroll
        for (int c = 4; c < kBN; c += 4) {
          mx0 = fmaxf(mx0, __uint_as_float(sr[c]));
          mx1 = fmaxf(mx1, __uint_as_float(sr[c + 1]));
          mx2 = fmaxf(mx2, __uint_as_float(sr[c + 2]));
          mx3 = fmaxf(mx3, __uint_as_float(sr[c + 3]));
        }
        const float m_new = fmaxf(m_run, fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2);
        if (j == 0) {
          m_run = m_new;
        } else if (__any_sync(0xffffffffu, m_new > m_run)) {
          // the warp moves its reference maxima; O (complete up to tile j-1) is rescaled
          const float alpha = m_run == -INFINITY ? 0.f : fast_exp2(m_run - m_new);
          if (!__all_sync(0xffffffffu, mbar_wait(bar(Bars::pv_done + t), (j - 1) & 1, &s_abort, prm.status))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D; c += 32) {         // 32 columns at a time: S stays in registers
            float o[32];
            tmem_ld32(tO(t) + lane_off + c, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tO(t) + lane_off + c, o);
          }
          l_run *= alpha;
          m_run = m_new;
        }
        lt = exp_pass(m_run == -INFINITY ? 0.f : m_run);
      }
      l_run += lt;
      tmem_st64(tS(t) + lane_off, pk);            // P_t(j) over the first 64 columns of S_t
      tc_fence_before();
      mbar_arrive(bar(Bars::p_full + t));
    }
    // ---- epilogue ------------------------------------------------------------------------
    if (ok && ntiles > 0) ok = mbar_wait(bar(Bars::pv_done + t), (ntiles - 1) & 1, &s_abort, prm.status);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    if (kClu && ok) {
      // Split-key partials: every CTA of the cluster stages its unnormalised O
      // rows and (m, l) in its own K/V ring region (free once its last P V has
      // completed: the K ring holds tile 0's rows, the V ring tile 1's), chunks
      // rotated by row so the 16-byte stores of a warp hit distinct banks. The
      // merge runs after the cluster barrier below.
      constexpr int kChunks = D / 4;
      const int srow = t * kBM + r;
      float4* stage = reinterpret_cast<float4*>(gbase + L::kK);
      float2* ml = reinterpret_cast<float2*>(gbase + L::kList);
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        float o[32];
        tmem_ld32(tO(t) + lane_off + c, o);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          stage[srow * kChunks + (c / 4 + q + r) % kChunks] =
              make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
      }
      ml[srow] = make_float2(m_run, l_run);
    } else if (ok) {
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      if (prm.nsplit > 1) {
        // partial result of this key range: normalised fp32 row + its log-sum-exp
        const int64_t prow = (static_cast<int64_t>(blockIdx.z) * p.cap + row) * p.H + h;
        float4* frow = reinterpret_cast<float4*>(prm.o_part + prow * D);
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          float o[32];
          if (ntiles > 0) tmem_ld32(tO(t) + lane_off + c, o);
          else
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = 0.f;
          if (valid) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              frow[c / 4 + q] = make_float4(o[4 * q] * inv, o[4 * q + 1] * inv, o[4 * q + 2] * inv, o[4 * q + 3] * inv);
          }
        }
        if (valid) prm.lse_part[prow] = l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
      } else {
        uint4* orow = reinterpret_cast<uint4*>(p.o + (row * p.H + h) * D);
  #pragma unroll
        for (int c = 0; c < D; c += 32) {
          float o[32];
          if (ntiles > 0) tmem_ld32(tO(t) + lane_off + c, o);
          else
  #pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = 0.f;
          if (valid) {
  #pragma unroll
            for (int q = 0; q < 4; ++q)
              orow[c / 8 + q] = make_uint4(pack_bf16x2(o[8 * q + 0] * inv, o[8 * q + 1] * inv),
                                           pack_bf16x2(o[8 * q + 2] * inv, o[8 * q + 3] * inv),
                                           pack_bf16x2(o[8 * q + 4] * inv, o[8 * q + 5] * inv),
                                           pack_bf16x2(o[8 * q + 6] * inv, o[8 * q + 7] * inv));
          }
        }
        if (valid && p.lse) p.lse[row * p.H + h] = l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
      }
    }
  };
  // the common tail; each warpgroup runs its own copy, so its CTA and cluster barriers
  // are the non-aligned forms
  auto tail = [&]() {
  // ---- split-key merge inside the cluster ------------------------------------------------
  // After every CTA has staged its partials (cluster barrier, release/acquire at
  // cluster scope), CTA rank k merges rows [k*R, (k+1)*R) of the 256, R =
  // ceil(256/S), reading every rank's staged rows over distributed shared
  // memory: two threads per row, each half a row. The second barrier keeps
  // every CTA's shared memory valid until its peers have read it.
  if constexpr (kClu) {
    cta_sync<true>();                                   // warps converged for the aligned barrier
    cluster_sync<true>();
    constexpr int kChunks = D / 4;
    const int S = prm.cluster;
    const int R = (kQT * kBM + S - 1) / S;
    const uint32_t crank = cluster_ctarank();
    const int srow = static_cast<int>(crank) * R + (tid >> 1);
    const int half = tid & 1;
    if (tid < 2 * R && srow < kQT * kBM && !s_abort) {
      const int r = srow % kBM;
      const int64_t row = row0 + srow;
      const bool valid = row < rows;
      float mk[kMaxCluster], ak[kMaxCluster];
      uint32_t sbase_k[kMaxCluster];
      float M = -INFINITY;
#pragma unroll
      for (int k = 0; k < kMaxCluster; ++k) {
        mk[k] = -INFINITY;
        ak[k] = 0.f;
        sbase_k[k] = 0u;
        if (k < S) {
          const float2 v = ld_cluster_f2(map_to_rank(smem_u32(gbase + L::kList) + 8u * srow, k));
          mk[k] = v.x;
          ak[k] = v.y;                                                  // l of rank k, for now
          sbase_k[k] = map_to_rank(smem_u32(gbase + L::kK), k);
          M = fmaxf(M, v.x);
        }
      }
      float l = 0.f;
#pragma unroll
      for (int k = 0; k < kMaxCluster; ++k) {
        const float lk = ak[k];
        ak[k] = mk[k] == -INFINITY ? 0.f : fast_exp2(mk[k] - M);
        l += ak[k] * lk;
      }
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint4* orow = reinterpret_cast<uint4*>(p.o + (row * p.H + h) * D) + half * (D / 16);
#pragma unroll
      for (int c8 = 0; c8 < D / 16; ++c8) {              // 8 columns per 16-byte output vector
        float o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = 0.f;
#pragma unroll
        for (int k = 0; k < kMaxCluster; ++k) {
          if (k >= S) break;
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int chunk = half * (kChunks / 2) + c8 * 2 + q;
            const float4 x = ld_cluster_f4(sbase_k[k] + static_cast<uint32_t>(srow * kChunks + (chunk + r) % kChunks) * 16u);
            o[4 * q] = fmaf(ak[k], x.x, o[4 * q]);
            o[4 * q + 1] = fmaf(ak[k], x.y, o[4 * q + 1]);
            o[4 * q + 2] = fmaf(ak[k], x.z, o[4 * q + 2]);
            o[4 * q + 3] = fmaf(ak[k], x.w, o[4 * q + 3]);
          }
        }
        if (valid)
          orow[c8] = make_uint4(pack_bf16x2(o[0] * inv, o[1] * inv), pack_bf16x2(o[2] * inv, o[3] * inv),
                                pack_bf16x2(o[4] * inv, o[5] * inv), pack_bf16x2(o[6] * inv, o[7] * inv));
      }
      if (valid && half == 0 && p.lse) p.lse[row * p.H + h] = l > 0.f ? (M + __log2f(l)) * kLn2 : -INFINITY;
    }
    cta_sync<true>();
    cluster_sync<true>();
  }

  // ---- teardown ------------------------------------------------------------------------
  if (warp == kMmaWarp && lane == 0) drain_wait(bar(Bars::drain), 0);   // no MMA may still write TMEM
  tc_fence_before();
  cta_sync<true>();
  tc_fence_after();
  if (warp == kMmaWarp) {
    __syncwarp();
    tmem_dealloc<kTmemCols>(tmem);
  }
  };
  // the producer warpgroup (TMA, MMA and two idle warps) hands registers to the two
  // softmax warpgroups; each side then runs to the end on its own (ptxas allots a
  // region the registers of its setmaxnreg only if the region does not rejoin the
  // other warps' code)
  if (warp >= kTmaWarp) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
    if (warp == kTmaWarp) tma_role();
    else if (warp == kMmaWarp) mma_role();
    tail();
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    softmax_role();
    tail();
  }
}

// Block mode (a key-block mask is given): tile t of CTA x holds the active rows
// of original query block qb = 2x + t -- the run of the ascending idx inside
// [128 qb, 128 qb + 128) -- and streams only the key tiles that block keeps, so
// every key tile a tile loads is work for all its rows. The two tiles' K and V
// loads interleave in the rings: (j, 0), (j, 1), (j + 1, 0), ..., skipping a
// tile whose list has ended; each stage has one reader, its own tile.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_blk_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, TcParams prm) {
  using L = Layout<D, kQT>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_ntiles[kQT];
  __shared__ int s_nrows[kQT];
  __shared__ int s_row0[kQT];
  __shared__ volatile int s_abort;
  __shared__ unsigned int s_wcnt[kQT][kThreads / 32];

  const AttnArgs& p = prm.a;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  const int64_t rows = active_count(p.count, p.cap);

  // ---- the query rows of each tile ------------------------------------------------------
  {
    if (warp == 0) {
      // lane 2t: first row of tile t; lane 2t + 1: one past its last row (lower bounds in idx)
      const int64_t key = (2 * static_cast<int64_t>(blockIdx.x) + (lane >> 1) + (lane & 1)) * 128;
      int64_t lo = 0, hi = rows;
      while (lo < hi) {
        const int64_t mid = (lo + hi) >> 1;
        if (p.idx[mid] < key) lo = mid + 1;
        else hi = mid;
      }
      const int64_t end = __shfl_down_sync(0xffffffffu, lo, 1);
      if (lane < 2 * kQT && (lane & 1) == 0) {
        const int64_t n = end - lo;
        s_row0[lane >> 1] = static_cast<int>(lo);
        s_nrows[lane >> 1] = static_cast<int>(n < 0 ? 0 : (n > kBM ? kBM : n));
      }
    }
    __syncthreads();
    if (s_nrows[0] == 0 && s_nrows[1] == 0) return;   // uniform: before TMEM or barriers
  }

  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - smem_u32(smem_raw));
  uint16_t* sList = reinterpret_cast<uint16_t*>(gbase + L::kList);   // [tile][kListMax]
  const uint32_t bar0 = sbase + L::kBar;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };

  // ---- setup: barriers, TMEM, key-tile lists ------------------------------------------
  if (tid == 0) {
    s_abort = 0;
    for (int t = 0; t < kQT; ++t) {
      mbar_init(bar(Bars::q_full + t), 1);
      mbar_init(bar(Bars::s_full + t), 1);
      mbar_init(bar(Bars::p_full + t), kBM);
      mbar_init(bar(Bars::pv_done + t), 1);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(Bars::k_full + s), 1);
      mbar_init(bar(Bars::v_full + s), 1);
      mbar_init(bar(Bars::k_empty + s), 1);
      mbar_init(bar(Bars::v_empty + s), 1);
    }
    mbar_init(bar(Bars::drain), 1);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tmem_alloc<kTmemCols>(smem_u32(&s_tmem));
  if (warp == kTmaWarp && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  {
    // tile t's key list: the key blocks its query block keeps, ascending
    int base[kQT] = {0, 0};
    const uint8_t* mrow[kQT];
    for (int t = 0; t < kQT; ++t)
      mrow[t] = p.bm + (2 * static_cast<int64_t>(blockIdx.x) + t) * p.nb;
    for (int kb0 = 0; kb0 < p.nb; kb0 += kThreads) {
      const int kb = kb0 + tid;
      unsigned int m[kQT];
      for (int t = 0; t < kQT; ++t) {
        const bool keep = s_nrows[t] > 0 && kb < p.nb && mrow[t][kb] != 0;
        m[t] = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) s_wcnt[t][warp] = __popc(m[t]);
      }
      __syncthreads();
      for (int t = 0; t < kQT; ++t) {
        int off = base[t], tot = 0;
        for (int i = 0; i < kThreads / 32; ++i) {
          off += i < warp ? s_wcnt[t][i] : 0;
          tot += s_wcnt[t][i];
        }
        if ((m[t] >> lane) & 1u)
          sList[t * L::kListMax + off + __popc(m[t] & ((1u << lane) - 1u))] = static_cast<uint16_t>(kb);
        base[t] += tot;
      }
      __syncthreads();
    }
    if (tid < kQT) s_ntiles[tid] = base[tid];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  auto tS = [&](int t) { return tmem + 256u * t; };          // S_t, later P_t (bf16 pairs)
  auto tO = [&](int t) { return tmem + 256u * t + 128u; };   // O_t accumulator
  auto tile_kb = [&](int t, int j) -> int { return static_cast<int>(sList[t * L::kListMax + j]); };
  const int n0 = s_ntiles[0], n1 = s_ntiles[1];
  // position of (tile t, key step j) in the K and V load sequence
  auto seq_of = [&](int j, int t) -> int {
    return (j < n0 ? j : n0) + (j < n1 ? j : n1) + (t == 1 && j < n0 ? 1 : 0);
  };

  auto tma_role = [&]() {
    // ================================ TMA producer =====================================
    if (lane == 0) {
      int issued_k = 0, issued_v = 0;
      bool q_issued[kQT];
      for (int t = 0; t < kQT; ++t) {
        q_issued[t] = s_ntiles[t] > 0;
        if (!q_issued[t]) continue;
        mbar_expect_tx(bar(Bars::q_full + t), L::kSub * kSubBytes);
        for (int s = 0; s < L::kSub; ++s)
          tma_load_3d(sbase + L::kQ + (t * L::kSub + s) * kSubBytes, &tmQ, 64 * s, h, s_row0[t],
                      bar(Bars::q_full + t));
      }
      // K and V stages are freed separately: a K stage as soon as the last S MMA
      // reading it completes (about one period before its PV stage), so the next
      // K tile streams in while the current P.V products still run.
      const int jmax = n0 > n1 ? n0 : n1;
      bool ok = true;
      for (int j = 0; ok && j < jmax; ++j) {
        for (int t = 0; ok && t < kQT; ++t) {
          if (j >= s_ntiles[t]) continue;
          const int q = seq_of(j, t);
          const int st = q % kStages;
          const uint32_t ph = ((q / kStages) - 1) & 1;
          const int key0 = tile_kb(t, j) * kBN;
          if (q >= kStages && !mbar_wait(bar(Bars::k_empty + st), ph, &s_abort, prm.status)) ok = false;
          if (!ok) break;
          mbar_expect_tx(bar(Bars::k_full + st), L::kSub * kSubBytes);
          for (int s = 0; s < L::kSub; ++s)
            tma_load_3d(sbase + L::kK + (st * L::kSub + s) * kSubBytes, &tmK, 64 * s, h, key0, bar(Bars::k_full + st));
          issued_k = q + 1;
          if (q >= kStages && !mbar_wait(bar(Bars::v_empty + st), ph, &s_abort, prm.status)) ok = false;
          if (!ok) break;
          mbar_expect_tx(bar(Bars::v_full + st), L::kSub * kSubBytes);
          for (int s = 0; s < L::kSub; ++s)
            tma_load_3d(sbase + L::kV + (st * L::kSub + s) * kSubBytes, &tmV, 64 * s, h, key0, bar(Bars::v_full + st));
          issued_v = q + 1;
        }
      }
      // drain: every load issued above must land before the CTA may exit
      for (int t = 0; t < kQT; ++t)
        if (q_issued[t]) drain_wait(bar(Bars::q_full + t), 0);
      for (int q = issued_k > kStages ? issued_k - kStages : 0; q < issued_k; ++q)
        drain_wait(bar(Bars::k_full + q % kStages), (q / kStages) & 1);
      for (int q = issued_v > kStages ? issued_v - kStages : 0; q < issued_v; ++q)
        drain_wait(bar(Bars::v_full + q % kStages), (q / kStages) & 1);
    }
  };
  auto mma_role = [&]() {
    // ================================ MMA issuer =======================================
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16(kBM, kBN, false, false);  // Q K^T: both K-major
      constexpr uint32_t kIdescO = idesc_bf16(kBM, D, false, true);     // P V: V is MN-major
      auto issue_s = [&](int t, int j) {
        const int st = seq_of(j, t) % kStages;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kSubBytes + (kk & 3) * 32;   // 16 bf16 along d
          const uint64_t da = sdesc_sw128(sbase + L::kQ + t * L::kSub * kSubBytes + off, 16, 1024);
          const uint64_t db = sdesc_sw128(sbase + L::kK + st * L::kSub * kSubBytes + off, 16, 1024);
          mma_f16_ss(tS(t), da, db, kIdescS, kk > 0);
        }
        mma_commit(bar(Bars::s_full + t));
        mma_commit(bar(Bars::k_empty + st));           // the one reader of this K stage
      };
      auto wait_k = [&](int t, int j) -> bool {
        const int q = seq_of(j, t);
        const bool r = mbar_wait(bar(Bars::k_full + q % kStages), (q / kStages) & 1, &s_abort, prm.status);
        tc_fence_after();
        return r;
      };
      bool ok = true;
      for (int t = 0; ok && t < kQT; ++t) {
        if (s_ntiles[t] == 0) continue;
        ok = wait_k(t, 0) && mbar_wait(bar(Bars::q_full + t), 0, &s_abort, prm.status);
        tc_fence_after();
        if (ok) issue_s(t, 0);
      }
      const int jmax = n0 > n1 ? n0 : n1;
      for (int j = 0; ok && j < jmax; ++j) {
        for (int t = 0; ok && t < kQT; ++t) {
          if (j >= s_ntiles[t]) continue;
          const int q = seq_of(j, t);
          const int st = q % kStages;
          ok = mbar_wait(bar(Bars::p_full + t), j & 1, &s_abort, prm.status);
          if (ok) ok = mbar_wait(bar(Bars::v_full + st), (q / kStages) & 1, &s_abort, prm.status);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            // B = V [128 keys x D], MN-major: 16 keys = 2 swizzle atoms of 8 rows;
            // LBO = next 64-wide d sub-tile, SBO = next 8 keys. A = P_t from TMEM,
            // 16 keys = 8 columns of bf16 pairs.
            const uint64_t db = sdesc_sw128(sbase + L::kV + st * L::kSub * kSubBytes + kk * 16 * 128, kSubBytes, 1024);
            mma_f16_ts(tO(t), tS(t) + 8 * kk, db, kIdescO, (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar(Bars::pv_done + t));
          mma_commit(bar(Bars::v_empty + st));         // the one reader of this V stage
          if (j + 1 < s_ntiles[t]) {
            // S_t(j+1) overwrites the columns P_t(j) was read from: tcgen05.mma
            // operations of one thread execute in issue order.
            ok = wait_k(t, j + 1);
            if (ok) issue_s(t, j + 1);
          }
        }
      }
      mma_commit(bar(Bars::drain));   // fires once every MMA issued above has completed
    }
  };
  auto softmax_role = [&]() {
    // ================================ softmax warps ====================================
    const int t = warp >> 2;                      // query tile of this warpgroup
    const int r = (warp & 3) * 32 + lane;         // row within the tile == TMEM lane
    const int64_t row = static_cast<int64_t>(s_row0[t]) + r;
    const bool valid = r < s_nrows[t];
    const int ntiles = s_ntiles[t];
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float sl2 = prm.scale_log2;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      // every wait result is made warp-uniform: tcgen05.ld/st are .sync.aligned
      if (!__all_sync(0xffffffffu, mbar_wait(bar(Bars::s_full + t), j & 1, &s_abort, prm.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int64_t key0 = static_cast<int64_t>(tile_kb(t, j)) * kBN;
      // a row outside the tile's query rows takes no key (its S is whatever the
      // padding rows held); keys past N are masked
      const int nvalid = valid ? static_cast<int>(p.N - key0 < kBN ? p.N - key0 : kBN) : 0;
      uint32_t sr[kBN];
      auto load_s = [&]() {
        tmem_ld128(tS(t) + lane_off, sr);
        if (nvalid < kBN) {
#pragma unroll
          for (int c = 0; c < kBN; ++c)
            if (c >= nvalid) sr[c] = __float_as_uint(-INFINITY);
        }
      };
      uint32_t pk[kBN / 2];
      // P = exp2(S * scale_log2 - base) as bf16 pairs into pk; returns the row sum of this tile
      auto exp_pass = [&](float base) -> float { return exp_row<kBN>(sr, sl2x2, base, pk); };
      load_s();
      // Fast path: keep the running reference max and skip the row max. Softmax is
      // exact for any reference; the tile's sum bounds every P, so P stays finite
      // and well inside bf16/fp32 range while the sum is at most kSumLimit.
      bool slow = j == 0;
      float lt = 0.f;
      if (!slow) {
        const float base = m_run == -INFINITY ? 0.f : m_run;
        lt = exp_pass(base);
        slow = __any_sync(0xffffffffu, !(lt <= kSumLimit));
        if (slow) load_s();                         // S is intact: P has not been stored yet
        else m_run = base;                          // a row with only masked keys so far now uses 0
      }
      if (slow) {
        float mx0 = __uint_as_float(sr[0]), mx1 = __uint_as_float(sr[1]);
        float mx2 = __uint_as_float(sr[2]), mx3 = __uint_as_float(sr[3]);
#pragma unroll
        for (int c = 4; c < kBN; c += 4) {
          mx0 = fmaxf(mx0, __uint_as_float(sr[c]));
          mx1 = fmaxf(mx1, __uint_as_float(sr[c + 1]));
          mx2 = fmaxf(mx2, __uint_as_float(sr[c + 2]));
          mx3 = fmaxf(mx3, __uint_as_float(sr[c + 3]));
        }
        const float m_new = fmaxf(m_run, fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2);
        if (j == 0) {
          m_run = m_new;
        } else if (__any_sync(0xffffffffu, m_new > m_run)) {
          // the warp moves its reference maxima; O (complete up to tile j-1) is rescaled
          const float alpha = m_run == -INFINITY ? 0.f : fast_exp2(m_run - m_new);
          if (!__all_sync(0xffffffffu, mbar_wait(bar(Bars::pv_done + t), (j - 1) & 1, &s_abort, prm.status))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D; c += 32) {         // 32 columns at a time: S stays in registers
            float o[32];
            tmem_ld32(tO(t) + lane_off + c, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tO(t) + lane_off + c, o);
          }
          l_run *= alpha;
          m_run = m_new;
        }
        lt = exp_pass(m_run == -INFINITY ? 0.f : m_run);
      }
      l_run += lt;
      tmem_st64(tS(t) + lane_off, pk);            // P_t(j) over the first 64 columns of S_t
      tc_fence_before();
      mbar_arrive(bar(Bars::p_full + t));
    }
    // ---- epilogue ------------------------------------------------------------------------
    if (ok && ntiles > 0) ok = mbar_wait(bar(Bars::pv_done + t), (ntiles - 1) & 1, &s_abort, prm.status);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    if (ok) {
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      {
        uint4* orow = reinterpret_cast<uint4*>(p.o + (row * p.H + h) * D);
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          float o[32];
          if (ntiles > 0) tmem_ld32(tO(t) + lane_off + c, o);
          else
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = 0.f;
          if (valid) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              orow[c / 8 + q] = make_uint4(pack_bf16x2(o[8 * q + 0] * inv, o[8 * q + 1] * inv),
                                           pack_bf16x2(o[8 * q + 2] * inv, o[8 * q + 3] * inv),
                                           pack_bf16x2(o[8 * q + 4] * inv, o[8 * q + 5] * inv),
                                           pack_bf16x2(o[8 * q + 6] * inv, o[8 * q + 7] * inv));
          }
        }
        if (valid && p.lse) p.lse[row * p.H + h] = l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
      }
    }
  };
  // the common tail; each warpgroup runs its own copy (non-aligned barrier)
  auto tail = [&]() {
  // ---- teardown ------------------------------------------------------------------------
  if (warp == kMmaWarp && lane == 0) drain_wait(bar(Bars::drain), 0);   // no MMA may still write TMEM
  tc_fence_before();
  cta_sync<true>();
  tc_fence_after();
  if (warp == kMmaWarp) {
    __syncwarp();
    tmem_dealloc<kTmemCols>(tmem);
  }
  };
  // registers from the producer warpgroup to the softmax warpgroups (as in attn_tc_kernel)
  if (warp >= kTmaWarp) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
    if (warp == kTmaWarp) tma_role();
    else if (warp == kMmaWarp) mma_role();
    tail();
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    softmax_role();
    tail();
  }
}

// ---- block mode, transposed products (d = 128) ------------------------------------------------
// A query block keeps few of its 128 tokens active (about 51 at 40% kept), so an M = 128 tile of
// query rows is mostly padding. Here the 128 keys of a key tile are the MMA's M and a unit of at
// most 64 active rows of one query block is its N:
//   S^T  = K Q^T     [128 keys x 64 rows]:     A = K tile (K-major), B = Q rows (K-major)
//   O^T += V^T P^T   [128 channels x 64 rows]: A = V tile read MN-major, B = P^T (MN-major)
// CTA (x, h, z) takes rows [64z, 64z + 64) of the active runs of query blocks 2x and 2x + 1 as
// units 0 and 1, one after the other: one stream of key tiles g = 0, 1, ... (unit 0's list, then
// unit 1's) through two-stage K and V rings. S^T and P^T are double-buffered (TMEM and shared
// memory), so the MMAs of tiles g + 2 and g overlap the softmax of tile g + 1.
// Four softmax warpgroups split a tile's 64 columns: warpgroup w takes columns [16w, 16w + 16);
// thread r of it owns key r of S^T (TMEM lane r) and channel r of O^T. The reference maximum is
// one per column (query row), shared by the 128 key threads of its warpgroup: after a unit's
// first key tile it changes only when an exponent argument exceeds kXLimit somewhere in the
// warpgroup's half of the tile, which one barrier reduction over the warpgroup decides. The two
// warpgroups share no barrier. The per-column sums stay in the key threads' registers and are
// reduced across threads once per unit.
// The single MMA-issuing thread is the pipeline's serial stage (each tcgen05.mma of N = 64 and
// each tcgen05.commit costs it tens of cycles), so it commits twice per tile: S^T(g)'s commit
// also frees K stage g % 2, and P V(g)'s commit frees V stage g % 2 and tells the softmax that
// O^T holds tile g.
namespace blkt {
constexpr int kUR = 64;                 // query rows per unit (MMA N)
constexpr int kWG = 4;                  // softmax warpgroups
constexpr int kCols = kUR / kWG;        // columns per softmax warpgroup
constexpr int kSmThreadsT = kWG * 128;  // softmax threads
// + one producer warpgroup (TMA warp, MMA warp, two idle warps). 20 warps leave 96 registers a
// thread, enough for a softmax thread's 16 columns, so the kernel needs no register split.
constexpr int kThreadsT = kSmThreadsT + 128;
constexpr int kTmaWarpT = kSmThreadsT / 32;
constexpr int kMmaWarpT = kTmaWarpT + 1;
constexpr int kQSub = kUR * 128;        // one [64 rows x 64 bf16] swizzled Q sub-tile
constexpr int kPTBytes = 128 * 128;     // P^T of one tile: 128 keys x 64 rows bf16 (one 128-byte row per key)
constexpr float kXLimit = 64.f;         // largest exponent argument (log2) kept without a new reference
constexpr int kTmemColsT = 256;         // S^T buffers at [0, 64) and [64, 128); O^T of unit u at [128 + 64u, +64)

struct LayoutT {
  static constexpr int kSub = 2;                                // d = 128: two 64-wide sub-tiles
  static constexpr int kQ = 0;                                  // [unit][sub] x kQSub
  static constexpr int kK = kQ + kQT * kSub * kQSub;            // [stage][sub] x kSubBytes
  static constexpr int kV = kK + kStages * kSub * kSubBytes;
  static constexpr int kPT = kV + kStages * kSub * kSubBytes;   // [buffer] x kPTBytes
  static constexpr int kRed = kPT + 2 * kPTBytes;               // float [warpgroup][warp][kCols]: column folds
  static constexpr int kRef = kRed + kWG * 4 * kCols * 4;       // float [kUR]: minus the reference (log2)
  static constexpr int kAux = kRef + kUR * 4;                   // float [kUR]: rescale factors, then 1/l
  static constexpr int kList = kAux + kUR * 4;                  // uint16 [unit][kListMax]: kept key blocks
  static constexpr int kListMax = 4096;
  static constexpr int kBar = kList + kQT * kListMax * 2;
  static constexpr int kBytes = kBar + 256;
  static constexpr int kAlloc = kBytes + 1024;
};
static_assert(LayoutT::kK % 1024 == 0 && LayoutT::kV % 1024 == 0 && LayoutT::kPT % 1024 == 0, "swizzle atoms");
static_assert(LayoutT::kAlloc <= 227 * 1024, "shared memory");

static_assert(kStages == 2, "S^T buffer g % 2 and K stage g % 2 share their barrier");
struct BarsT {  // mbarrier indices (8 bytes each)
  static constexpr int q_full = 0;                     // + unit
  static constexpr int k_full = q_full + kQT;          // + stage
  static constexpr int v_full = k_full + kStages;      // + stage
  static constexpr int s_full = v_full + kStages;      // + g % 2: S^T(g) complete, K stage g % 2 free
  static constexpr int pv_done = s_full + 2;           // + g % 2: P V(g) complete, V stage g % 2 free
  static constexpr int p_full = pv_done + 2;           // + g % 2: P^T(g) written (every softmax thread)
  static constexpr int drain = p_full + 2;             // last commit of the MMA thread
  static constexpr int count = drain + 1;
};
static_assert(BarsT::count * 8 <= 256, "barrier block");

__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// Barrier of one softmax warpgroup (named barrier `id`, 128 threads).
__device__ __forceinline__ void wg_sync(int id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }
// Barrier of one softmax warpgroup that also returns the OR of `pred` over its 128 threads.
__device__ __forceinline__ bool wg_any(int id, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n.reg .pred p, q;\nsetp.ne.u32 p, %1, 0;\nbar.red.or.pred q, %2, 128, p;\nselp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id)
      : "memory");
  return r != 0;
}
// Shared-memory descriptor (128-byte swizzle, SBO 1024) as two 32-bit words: lo = start address
// >> 4 | LBO >> 4 << 16, hi = SBO >> 4 | version | swizzle mode. Adding (offset >> 4) to lo moves
// the start address (shared addresses stay below 2^18, so the 14-bit field cannot carry).
__host__ __device__ constexpr uint32_t sdesc_lo(uint32_t saddr, uint32_t lbo) { return (saddr >> 4) | ((lbo >> 4) << 16); }
constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
__device__ __forceinline__ void mma_ss_words(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\n.reg .b64 da, db;\nsetp.ne.b32 p, %4, 0;\nmov.b64 da, {%1, %5};\nmov.b64 db, {%2, %5};\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, p;\n}\n"
      ::"r"(d_tmem), "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(accumulate), "r"(kDescHi)
      : "memory");
}
// Folds kN per-thread column values across the warp's 32 lanes by recursive halving (max or
// sum); afterwards lane l holds the warp's result for column l / (32 / kN) in v[0].
template <int kN, bool kMax>
__device__ __forceinline__ void warp_fold(float (&v)[kN], int lane) {
#pragma unroll
  for (int s = 0; s < 5; ++s) {
    const int o = 16 >> s, n = kN >> s;
    if (n >= 2) {
      const bool up = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < n / 2; ++i) {
        const float send = up ? v[i] : v[i + n / 2];
        const float keep = up ? v[i + n / 2] : v[i];
        const float got = __shfl_xor_sync(0xffffffffu, send, o);
        v[i] = kMax ? fmaxf(keep, got) : keep + got;
      }
    } else {   // lanes l and l ^ o hold the same column
      const float got = __shfl_xor_sync(0xffffffffu, v[0], o);
      v[0] = kMax ? fmaxf(v[0], got) : v[0] + got;
    }
  }
}
}  // namespace blkt

__global__ void __launch_bounds__(blkt::kThreadsT, 1)
attn_blkt_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, TcParams prm) {
  using namespace blkt;
  constexpr int D = 128;
  using L = LayoutT;
  using B = BarsT;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_ntiles[kQT];
  __shared__ int s_nrows[kQT];
  __shared__ int s_row0[kQT];
  __shared__ volatile int s_abort;
  __shared__ unsigned int s_wcnt[kQT][kThreadsT / 32];

  const AttnArgs& p = prm.a;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  const int64_t rows = active_count(p.count, p.cap);

  // ---- the query rows of each unit --------------------------------------------------------
  {
    if (warp == 0) {
      // lane 2u: first row of query block 2x + u; lane 2u + 1: one past its last (lower bounds in idx)
      const int64_t key = (2 * static_cast<int64_t>(blockIdx.x) + (lane >> 1) + (lane & 1)) * 128;
      int64_t lo = 0, hi = rows;
      while (lo < hi) {
        const int64_t mid = (lo + hi) >> 1;
        if (p.idx[mid] < key) lo = mid + 1;
        else hi = mid;
      }
      const int64_t end = __shfl_down_sync(0xffffffffu, lo, 1);
      if (lane < 2 * kQT && (lane & 1) == 0) {
        const int64_t r0 = lo + static_cast<int64_t>(kUR) * blockIdx.z;
        const int64_t n = end - r0;
        s_row0[lane >> 1] = static_cast<int>(r0 < rows ? r0 : rows);
        s_nrows[lane >> 1] = static_cast<int>(n < 0 ? 0 : (n > kUR ? kUR : n));
      }
    }
    __syncthreads();
    if (s_nrows[0] == 0 && s_nrows[1] == 0) return;   // uniform: before TMEM or barriers
  }

  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - smem_u32(smem_raw));
  uint16_t* sList = reinterpret_cast<uint16_t*>(gbase + L::kList);   // [unit][kListMax]
  const uint32_t bar0 = sbase + L::kBar;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };

  // ---- setup: barriers, TMEM, key-tile lists ------------------------------------------------
  if (tid == 0) {
    s_abort = 0;
    for (int u = 0; u < kQT; ++u) mbar_init(bar(B::q_full + u), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(B::k_full + s), 1);
      mbar_init(bar(B::v_full + s), 1);
      mbar_init(bar(B::s_full + s), 1);
      mbar_init(bar(B::pv_done + s), 1);
      mbar_init(bar(B::p_full + s), kSmThreadsT);
    }
    mbar_init(bar(B::drain), 1);
    fence_mbar_init();
  }
  if (warp == kMmaWarpT) tmem_alloc<kTmemColsT>(smem_u32(&s_tmem));
  if (warp == kTmaWarpT && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  {
    // unit u's key list: the key blocks its query block keeps, ascending
    int base[kQT] = {0, 0};
    const uint8_t* mrow[kQT];
    for (int u = 0; u < kQT; ++u)
      mrow[u] = p.bm + (2 * static_cast<int64_t>(blockIdx.x) + u) * p.nb;
    for (int kb0 = 0; kb0 < p.nb; kb0 += kThreadsT) {
      const int kb = kb0 + tid;
      unsigned int m[kQT];
      for (int u = 0; u < kQT; ++u) {
        const bool keep = s_nrows[u] > 0 && kb < p.nb && mrow[u][kb] != 0;
        m[u] = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) s_wcnt[u][warp] = __popc(m[u]);
      }
      __syncthreads();
      for (int u = 0; u < kQT; ++u) {
        int off = base[u], tot = 0;
        for (int i = 0; i < kThreadsT / 32; ++i) {
          off += i < warp ? s_wcnt[u][i] : 0;
          tot += s_wcnt[u][i];
        }
        if ((m[u] >> lane) & 1u)
          sList[u * L::kListMax + off + __popc(m[u] & ((1u << lane) - 1u))] = static_cast<uint16_t>(kb);
        base[u] += tot;
      }
      __syncthreads();
    }
    if (tid < kQT) s_ntiles[tid] = base[tid];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  auto tS = [&](int b) { return tmem + 64u * b; };           // S^T buffer b (fp32, 64 columns)
  auto tO = [&](int u) { return tmem + 128u + 64u * u; };    // O^T of unit u (fp32, 64 columns)
  const int n0 = s_ntiles[0], nt = n0 + s_ntiles[1];          // key tiles of unit 0, of both
  auto unit_of = [&](int g) { return g < n0 ? 0 : 1; };
  auto step_of = [&](int g) { return g < n0 ? g : g - n0; };  // position in its unit's list
  auto tile_kb = [&](int g) -> int { return static_cast<int>(sList[unit_of(g) * L::kListMax + step_of(g)]); };

  auto tma_role = [&]() {
    // ================================ TMA producer =====================================
    if (lane == 0) {
      int issued_k = 0, issued_v = 0;
      bool q_issued[kQT];
      for (int u = 0; u < kQT; ++u) {
        q_issued[u] = s_ntiles[u] > 0;
        if (!q_issued[u]) continue;
        mbar_expect_tx(bar(B::q_full + u), L::kSub * kQSub);
        for (int s = 0; s < L::kSub; ++s)
          tma_load_3d(sbase + L::kQ + (u * L::kSub + s) * kQSub, &tmQ, 64 * s, h, s_row0[u], bar(B::q_full + u));
      }
      // K and V stages are freed separately: K stage g % 2 when S^T(g) completes (two tiles
      // ahead of its P V), V stage g % 2 when P V(g) does
      for (int g = 0; g < nt; ++g) {
        const int st = g % kStages;
        const uint32_t ph = ((g / kStages) - 1) & 1;
        const int key0 = tile_kb(g) * kBN;
        if (g >= kStages && !mbar_wait(bar(B::s_full + st), ph, &s_abort, prm.status)) break;
        mbar_expect_tx(bar(B::k_full + st), L::kSub * kSubBytes);
        for (int s = 0; s < L::kSub; ++s)
          tma_load_3d(sbase + L::kK + (st * L::kSub + s) * kSubBytes, &tmK, 64 * s, h, key0, bar(B::k_full + st));
        issued_k = g + 1;
        if (g >= kStages && !mbar_wait(bar(B::pv_done + st), ph, &s_abort, prm.status)) break;
        mbar_expect_tx(bar(B::v_full + st), L::kSub * kSubBytes);
        for (int s = 0; s < L::kSub; ++s)
          tma_load_3d(sbase + L::kV + (st * L::kSub + s) * kSubBytes, &tmV, 64 * s, h, key0, bar(B::v_full + st));
        issued_v = g + 1;
      }
      // drain: every load issued above must land before the CTA may exit
      for (int u = 0; u < kQT; ++u)
        if (q_issued[u]) drain_wait(bar(B::q_full + u), 0);
      for (int g = issued_k > kStages ? issued_k - kStages : 0; g < issued_k; ++g)
        drain_wait(bar(B::k_full + g % kStages), (g / kStages) & 1);
      for (int g = issued_v > kStages ? issued_v - kStages : 0; g < issued_v; ++g)
        drain_wait(bar(B::v_full + g % kStages), (g / kStages) & 1);
    }
  };
  auto mma_role = [&]() {
    // ================================ MMA issuer =======================================
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16(kBN, kUR, false, false);  // K Q^T: both K-major
      constexpr uint32_t kIdescO = idesc_bf16(D, kUR, true, true);      // V^T P^T: both MN-major
      // descriptor words of the operand bases (LBO: 16 bytes for K-major operands; the next
      // 64-wide sub-tile for V^T, the next 64 rows for P^T, neither reached by N = 64 rows)
      const uint32_t k_lo = sdesc_lo(sbase + L::kK, 16), q_lo = sdesc_lo(sbase + L::kQ, 16);
      const uint32_t v_lo = sdesc_lo(sbase + L::kV, kSubBytes), pt_lo = sdesc_lo(sbase + L::kPT, kPTBytes);
      // S^T(g) = K_g Q_u^T into buffer g % 2
      auto issue_s = [&](int g) -> bool {
        const int st = g % kStages, u = unit_of(g);
        if (!mbar_wait(bar(B::k_full + st), (g / kStages) & 1, &s_abort, prm.status)) return false;
        if (step_of(g) == 0 && !mbar_wait(bar(B::q_full + u), 0, &s_abort, prm.status)) return false;
        tc_fence_after();
        const uint32_t a0 = k_lo + ((st * L::kSub * kSubBytes) >> 4), b0 = q_lo + ((u * L::kSub * kQSub) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // 16 channels: sub-tile kk / 4, 32-byte chunk kk % 4 of each 128-byte row
          mma_ss_words(tS(g & 1), a0 + (((kk >> 2) * kSubBytes + (kk & 3) * 32) >> 4),
                       b0 + (((kk >> 2) * kQSub + (kk & 3) * 32) >> 4), kIdescS, kk > 0);
        }
        mma_commit(bar(B::s_full + st));               // S^T(g) complete; K stage g % 2 free
        return true;
      };
      bool ok = true;
      for (int g = 0; ok && g < nt && g < 2; ++g) ok = issue_s(g);
      for (int g = 0; ok && g < nt; ++g) {
        const int st = g % kStages, u = unit_of(g), j = step_of(g);
        ok = mbar_wait(bar(B::p_full + st), (g >> 1) & 1, &s_abort, prm.status);
        if (ok) ok = mbar_wait(bar(B::v_full + st), (g / kStages) & 1, &s_abort, prm.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a0 = v_lo + ((st * L::kSub * kSubBytes) >> 4), b0 = pt_lo + ((st * kPTBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          // A = V^T [128 channels x 16 keys], MN-major: 16 keys = 2 swizzle atoms of 8 rows
          // (SBO), channels 64-127 in the next sub-tile (LBO). B = P^T [64 rows x 16 keys],
          // MN-major: one 64-row atom, 8 keys per SBO.
          mma_ss_words(tO(u), a0 + ((kk * 16 * 128) >> 4), b0 + ((kk * 16 * 128) >> 4), kIdescO,
                       (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(B::pv_done + st));              // P V(g) complete; V stage g % 2 free
        // S^T(g+2) reuses buffer g % 2: the softmax has read S^T(g), since P^T(g) is complete.
        // tcgen05.mma operations of one thread execute in issue order, so S^T(g+2)'s
        // completion also implies that P V(g) has finished reading P^T buffer g % 2.
        if (g + 2 < nt) ok = issue_s(g + 2);
      }
      mma_commit(bar(B::drain));   // fires once every MMA issued above has completed
    }
  };
  auto softmax_role = [&]() {
    // ================================ softmax warps ====================================
    const int w = warp >> 2;                       // column group of this warpgroup
    const int r = (warp & 3) * 32 + lane;          // key of S^T, channel of O^T == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int c0 = kCols * w;                      // first column (query row of the unit) of this group
    const int bid = 1 + w;                         // this warpgroup's named barrier
    float* red = reinterpret_cast<float*>(gbase + L::kRed) + w * 4 * kCols;
    float* nref = reinterpret_cast<float*>(gbase + L::kRef) + c0;
    float* aux = reinterpret_cast<float*>(gbase + L::kAux) + c0;
    const float sl2 = prm.scale_log2;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    const uint64_t zero2 = f2_pack(0.f, 0.f);
    // a unit with rows but no kept key block: zero output, log-sum-exp -inf
    for (int u = 0; u < kQT; ++u) {
      if (s_ntiles[u] > 0 || s_nrows[u] == 0) continue;
      const int64_t row0 = s_row0[u];
      for (int i = tid; i < s_nrows[u] * (D / 8); i += kSmThreadsT)
        *reinterpret_cast<uint4*>(p.o + ((row0 + i / (D / 8)) * p.H + h) * D + (i % (D / 8)) * 8) =
            make_uint4(0u, 0u, 0u, 0u);
      if (p.lse)
        for (int i = tid; i < s_nrows[u]; i += kSmThreadsT) p.lse[(row0 + i) * p.H + h] = -INFINITY;
    }
    uint64_t lsum[kCols / 2];                      // per-column partial sums over this thread's keys
#pragma unroll
    for (int i = 0; i < kCols / 2; ++i) lsum[i] = zero2;
    for (int g = 0; g < nt; ++g) {
      const int u = unit_of(g), j = step_of(g), b = g & 1;
      // every wait result is made warp-uniform: tcgen05.ld/st are .sync.aligned
      const bool w_ok = __all_sync(0xffffffffu, mbar_wait(bar(B::s_full + b), (g >> 1) & 1, &s_abort, prm.status));
      const bool kvalid = static_cast<int64_t>(tile_kb(g)) * kBN + r < p.N;   // keys past N are masked
      float sv[kCols];
      auto load_s = [&]() {
        tmem_ld16(tS(b) + lane_off + c0, sv);
        if (!kvalid) {
#pragma unroll
          for (int c = 0; c < kCols; ++c) sv[c] = -INFINITY;
        }
      };
      // exponent arguments x = S * scale_log2 - reference, in place; returns their maximum
      auto x_pass = [&]() -> float {
        float xm0 = -INFINITY, xm1 = -INFINITY;
#pragma unroll
        for (int c = 0; c < kCols; c += 4) {
          const float4 nr = *reinterpret_cast<const float4*>(nref + c);
          const uint64_t x01 = ffma2(f2_pack(sv[c], sv[c + 1]), sl2x2, f2_pack(nr.x, nr.y));
          const uint64_t x23 = ffma2(f2_pack(sv[c + 2], sv[c + 3]), sl2x2, f2_pack(nr.z, nr.w));
          f2_unpack(x01, sv[c], sv[c + 1]);
          f2_unpack(x23, sv[c + 2], sv[c + 3]);
          xm0 = fmax3f(xm0, sv[c], sv[c + 1]);
          xm1 = fmax3f(xm1, sv[c + 2], sv[c + 3]);
        }
        return fmaxf(xm0, xm1);
      };
      // P = 2^x in place (fp32) and as bf16 pairs
      uint32_t pk[kCols / 2];
      auto exp_pass = [&]() {
#pragma unroll
        for (int c = 0; c < kCols; c += 2) {
          sv[c] = fast_exp2(sv[c]);
          sv[c + 1] = fast_exp2(sv[c + 1]);
          pk[c >> 1] = pack_bf16x2(sv[c], sv[c + 1]);
        }
      };
      // Fast path: keep the references. Softmax is exact for any reference (the final l uses
      // the same one); while every argument is at most kXLimit, P and the sums stay finite.
      // The exponentials run before the warpgroup's vote and are discarded if it fails.
      bool slow = j == 0;
      if (w_ok) {
        tc_fence_after();
        load_s();
        if (!slow) {
          slow = !(x_pass() <= kXLimit);
          exp_pass();
        }
      }
      if (wg_any(bid, !w_ok || slow)) {
        if (wg_any(bid, !w_ok)) break;             // uniform over the warpgroup
        // new references: this tile's column maxima over the 128 keys
        if (j > 0) load_s();                       // S^T is intact: P^T(g) has not been released
        {
          float v[kCols];
#pragma unroll
          for (int c = 0; c < kCols; ++c) v[c] = sv[c];
          warp_fold<kCols, true>(v, lane);
          if ((lane & (32 / kCols - 1)) == 0) red[(warp & 3) * kCols + lane / (32 / kCols)] = v[0];
        }
        wg_sync(bid);
        if (r < kCols) {
          const float mx = fmaxf(fmaxf(red[r], red[kCols + r]), fmaxf(red[2 * kCols + r], red[3 * kCols + r])) * sl2;
          const float old = j == 0 ? -INFINITY : -nref[r];
          float mnew = fmaxf(old, mx);
          if (mnew == -INFINITY) mnew = 0.f;       // a column without a finite score keeps reference 0
          aux[r] = j == 0 ? 1.f : fast_exp2(old - mnew);
          nref[r] = -mnew;
        }
        wg_sync(bid);
        load_s();
        if (j > 0) {
          // O^T must hold every P V of this unit up to tile j-1 before it moves to the new
          // references (P V(g-1) was issued after S^T(g), so it may still run; P V(g-3) has
          // completed and P V(g+1) cannot start, so the parity names P V(g-1))
          const bool pv_ok = __all_sync(
              0xffffffffu, mbar_wait(bar(B::pv_done + ((g - 1) & 1)), ((g - 1) >> 1) & 1, &s_abort, prm.status));
          if (wg_any(bid, !pv_ok)) break;
          tc_fence_after();
          float o[kCols];
          tmem_ld16(tO(u) + lane_off + c0, o);
#pragma unroll
          for (int c = 0; c < kCols; c += 4) {
            const float4 al = *reinterpret_cast<const float4*>(aux + c);
            o[c] *= al.x;
            o[c + 1] *= al.y;
            o[c + 2] *= al.z;
            o[c + 3] *= al.w;
            lsum[c >> 1] = ffma2(lsum[c >> 1], f2_pack(al.x, al.y), zero2);
            lsum[(c >> 1) + 1] = ffma2(lsum[(c >> 1) + 1], f2_pack(al.z, al.w), zero2);
          }
          tmem_st16(tO(u) + lane_off + c0, o);
        }
        x_pass();
        exp_pass();
      }
      // per-column partial sums (this thread's one key of the tile)
#pragma unroll
      for (int c = 0; c < kCols; c += 2) lsum[c >> 1] = fadd2(lsum[c >> 1], f2_pack(sv[c], sv[c + 1]));
      // this group's part of key r's row of P^T: 16-byte chunks 2w and 2w + 1, 128-byte swizzle
      // (chunk q at q ^ (r % 8))
      uint8_t* ptb = gbase + L::kPT + b * kPTBytes;
#pragma unroll
      for (int q = 0; q < kCols / 8; ++q)
        *reinterpret_cast<uint4*>(ptb + r * 128 + ((((kCols / 8) * w + q) ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      fence_proxy_async_smem();                    // the tensor core reads P^T through the async proxy
      tc_fence_before();
      mbar_arrive(bar(B::p_full + b));
      if (j == s_ntiles[u] - 1) {
        // ---- unit u complete: column sums, O^T / l, stores ------------------------------
        // P V(g), the unit's last (P V(g-2) has completed and P V(g+2) cannot start)
        const bool d_ok =
            __all_sync(0xffffffffu, mbar_wait(bar(B::pv_done + b), (g >> 1) & 1, &s_abort, prm.status));
        if (wg_any(bid, !d_ok)) break;
        tc_fence_after();
        {
          float v[kCols];
#pragma unroll
          for (int i = 0; i < kCols / 2; ++i) f2_unpack(lsum[i], v[2 * i], v[2 * i + 1]);
          warp_fold<kCols, false>(v, lane);
          if ((lane & (32 / kCols - 1)) == 0) red[(warp & 3) * kCols + lane / (32 / kCols)] = v[0];
        }
        wg_sync(bid);
        const int nrows = s_nrows[u];
        const int64_t row0 = s_row0[u];
        uint8_t* qbuf = gbase + L::kQ + u * L::kSub * kQSub;
        if (r < kCols) {
          const float l = (red[r] + red[kCols + r]) + (red[2 * kCols + r] + red[3 * kCols + r]);
          aux[r] = l > 0.f ? 1.f / l : 0.f;
          if (c0 + r < nrows && p.lse)
            p.lse[(row0 + c0 + r) * p.H + h] = l > 0.f ? (__log2f(l) - nref[r]) * kLn2 : -INFINITY;
        }
        wg_sync(bid);
        {
          // O^T / l, transposed through unit u's Q buffer (its last reader, S^T(g), has
          // completed): row c of the unit at c * 256 bytes; each warpgroup its own 16 rows
          float o[kCols];
          tmem_ld16(tO(u) + lane_off + c0, o);
          uint16_t* ot = reinterpret_cast<uint16_t*>(qbuf);
#pragma unroll
          for (int c = 0; c < kCols; c += 4) {
            const float4 inv = *reinterpret_cast<const float4*>(aux + c);
            const uint32_t w01 = pack_bf16x2(o[c] * inv.x, o[c + 1] * inv.y);
            const uint32_t w23 = pack_bf16x2(o[c + 2] * inv.z, o[c + 3] * inv.w);
            ot[(c0 + c) * D + r] = static_cast<uint16_t>(w01 & 0xffffu);
            ot[(c0 + c + 1) * D + r] = static_cast<uint16_t>(w01 >> 16);
            ot[(c0 + c + 2) * D + r] = static_cast<uint16_t>(w23 & 0xffffu);
            ot[(c0 + c + 3) * D + r] = static_cast<uint16_t>(w23 >> 16);
          }
        }
        wg_sync(bid);
        for (int i = r; i < kCols * (D / 8); i += kBM) {
          const int c = c0 + i / (D / 8), q = i % (D / 8);
          if (c < nrows)
            *reinterpret_cast<uint4*>(p.o + ((row0 + c) * p.H + h) * D + q * 8) =
                *reinterpret_cast<const uint4*>(qbuf + c * (D * 2) + q * 16);
        }
#pragma unroll
        for (int i = 0; i < kCols / 2; ++i) lsum[i] = zero2;
      }
    }
  };
  // the common tail; each warpgroup runs its own copy (non-aligned barrier)
  if (warp == kTmaWarpT) tma_role();
  else if (warp == kMmaWarpT) mma_role();
  else if (warp < kTmaWarpT) softmax_role();
  // ---- teardown ------------------------------------------------------------------------
  if (warp == kMmaWarpT && lane == 0) drain_wait(bar(B::drain), 0);   // no MMA may still write TMEM
  tc_fence_before();
  cta_sync<true>();
  tc_fence_after();
  if (warp == kMmaWarpT) {
    __syncwarp();
    tmem_dealloc<kTmemColsT>(tmem);
  }
}

// ---- host ------------------------------------------------------------------------------------
// [rows, H, d] bf16, token-major -> 3-D map (d, H, rows), box (64, 1, box_rows), 128-byte swizzle.
int make_map(EncodeTiledFn enc, CUtensorMap* m, const void* base, int64_t rows, int H, int d, int box_rows = 128) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H) * d * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TPS_ERR_CUDA, "pruned_attn: cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return TPS_OK;
}

// Sets the kernel's dynamic shared-memory limit once per device (setting it
// twice is harmless; devices numbered 64 and above set it on every launch).
template <auto kKernel>
int smem_attribute(int bytes) {
  static std::atomic<bool> done[64];   // one set per kernel
  int dev = 0;
  cudaGetDevice(&dev);
  const bool cached = dev >= 0 && dev < 64 && done[dev].load(std::memory_order_acquire);
  if (!cached) {
    cudaError_t e = cudaFuncSetAttribute(kKernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return cuda_status(e, "pruned_attn: smem attribute");
    if (dev >= 0 && dev < 64) done[dev].store(true, std::memory_order_release);
  }
  return TPS_OK;
}

// Dense: ceil(cap/256) x H x nsplit CTAs of two 128-row tiles of compacted rows.
// Masked (block mode): ceil(nb/2) x H CTAs, CTA x holding the active rows of
// query blocks 2x and 2x+1, each tile with its own key list; with d = 128 the
// transposed kernel, ceil(nb/2) x H x 2 CTAs (z: rows 0-63 or 64-127 of each run).
template <int D>
int launch(const AttnArgs& a, cudaStream_t st, int nsplit = 1, float* o_part = nullptr, float* lse_part = nullptr,
           int64_t tile0 = 0, int64_t ntiles = -1) {
  if (a.cap == 0) return TPS_OK;
  EncodeTiledFn enc;
  if (int e = tensor_map_encoder(&enc, "pruned_attn")) return e;
  int err;
  unsigned int* status = device_status(&err);
  if (!status) return err;
  CUtensorMap mq, mk, mv;
  if (int e = make_map(enc, &mq, a.q, a.cap, a.H, a.d)) return e;
  if (int e = make_map(enc, &mk, a.k, a.N, a.H, a.d)) return e;
  if (int e = make_map(enc, &mv, a.v, a.N, a.H, a.d)) return e;
  TcParams prm{a, a.scale * kLog2e, status, nsplit, o_part, lse_part, 1, static_cast<int>(tile0)};
  if (a.bm) {
    if constexpr (D == 128) {
      // transposed products: units of at most 64 rows of one query block, z = which 64 rows
      CUtensorMap mq64;
      if (int e = make_map(enc, &mq64, a.q, a.cap, a.H, a.d, blkt::kUR)) return e;
      constexpr int kSmem = blkt::LayoutT::kAlloc;
      if (int e = smem_attribute<attn_blkt_kernel>(kSmem)) return e;
      dim3 grid(static_cast<unsigned int>((a.nb + kQT - 1) / kQT), static_cast<unsigned int>(a.H), kBM / blkt::kUR);
      attn_blkt_kernel<<<grid, blkt::kThreadsT, kSmem, st>>>(mq64, mk, mv, prm);
    } else {
      constexpr int kSmem = Layout<D, kQT>::kAlloc;
      if (int e = smem_attribute<attn_blk_kernel<D>>(kSmem)) return e;
      dim3 grid(static_cast<unsigned int>((a.nb + kQT - 1) / kQT), static_cast<unsigned int>(a.H), 1u);
      attn_blk_kernel<D><<<grid, kThreads, kSmem, st>>>(mq, mk, mv, prm);
    }
  } else {
    constexpr int kSmem = Layout<D, 1>::kAlloc;
    if (int e = smem_attribute<attn_tc_kernel<D, false>>(kSmem)) return e;
    if (ntiles < 0) ntiles = (a.cap + kQT * kBM - 1) / (kQT * kBM);
    dim3 grid(static_cast<unsigned int>(ntiles), static_cast<unsigned int>(a.H), static_cast<unsigned int>(nsplit));
    attn_tc_kernel<D, false><<<grid, kThreads, kSmem, st>>>(mq, mk, mv, prm);
  }
  return launch_status("pruned_attn");
}

// CTAs of the dense kernel resident at once when launched in clusters of S
// along z: cudaOccupancyMaxActiveClusters x S (the SM count for S = 1),
// cached per device; 0 if clusters of S cannot be scheduled.
template <int D>
int cluster_slots(int S) {
  if (S <= 1) return sm_count();
  static std::atomic<int> cache[64][kMaxCluster + 1];   // 0 = not yet queried; stored as slots + 1
  int dev = 0;
  cudaGetDevice(&dev);
  const bool cacheable = dev >= 0 && dev < 64;
  if (cacheable) {
    const int v = cache[dev][S].load(std::memory_order_acquire);
    if (v > 0) return v - 1;
  }
  if (smem_attribute<attn_tc_kernel<D, true>>(Layout<D, 1>::kAlloc)) return 0;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(1, 1, static_cast<unsigned int>(S));
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Layout<D, 1>::kAlloc;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = static_cast<unsigned int>(S);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, attn_tc_kernel<D, true>, &cfg) != cudaSuccess) {
    cudaGetLastError();                 // a failed query leaves its error in the last-error slot
    n = 0;
  }
  const int slots = n * S;
  if (cacheable) cache[dev][S].store(slots + 1, std::memory_order_release);
  return slots;
}

// How a dense launch runs. The unit of work is one 256-row query tile pair of
// one head; an unsplit grid of U units on P SMs (one CTA each) takes
// ceil(U / P) unit times. Two ways out of a mostly empty last wave:
//  - the whole grid split S <= 4 ways along the keys, the S CTAs of a unit
//    forming a cluster along z that merges its partials over distributed shared
//    memory: ceil(U S / slots_S) / S unit times, slots_S = CTAs the GPU keeps
//    resident in clusters of S;
//  - the grid's full waves unsplit, then its remaining query tiles in a second
//    launch split S_t ways: those waves plus the split tail.
// A split pays its merge and cluster barriers (kSplitTax, measured on mid: 5%
// at equal wave counts) and a second launch its gap (kLaunchGap, in unit
// times); each split keeps >= 4 key tiles; a plan must gain 2% to be taken.
struct DensePlan {
  int split = 1;            // whole-grid key split (1: none)
  int64_t main_tiles = 0;   // tiles of the unsplit launch (all of them without a tail)
  int tail_split = 1;       // key split of the tail launch (1: no tail launch)
};
constexpr double kSplitTax = 1.06;
constexpr double kLaunchGap = 0.02;

template <int D>
DensePlan plan_dense(int64_t cap, int H, int64_t N) {
  DensePlan plan;
  const int64_t tiles = (cap + kQT * kBM - 1) / (kQT * kBM);
  plan.main_tiles = tiles;
  const int64_t units = tiles * H;
  const int64_t nkt = (N + kBN - 1) / kBN;
  const int64_t P = sm_count();
  if (units <= 0 || P <= 0) return plan;
  auto waves = [&](int64_t u, int S) -> double {   // unit times of u units split S ways
    const int64_t slots = S == 1 ? P : cluster_slots<D>(S);
    if (slots <= 0) return 1e30;
    return static_cast<double>((u * S + slots - 1) / slots) / S * (S > 1 ? kSplitTax : 1.0);
  };
  const double base = waves(units, 1);
  double best = base;
  for (int S = 2; S <= kMaxCluster && nkt >= 4 * S; ++S) {
    const double c = waves(units, S);
    if (c < best) {
      best = c;
      plan.split = S;
    }
  }
  const int64_t full = units / P;
  const int64_t t1 = full * P / H;                 // tiles that fit the full waves
  if (full >= 1 && t1 >= 1 && t1 < tiles) {
    const double main_cost = waves(t1 * H, 1) + kLaunchGap;
    const int64_t ut = (tiles - t1) * H;
    for (int S = 2; S <= kMaxCluster && nkt >= 4 * S; ++S) {
      const double c = main_cost + waves(ut, S);
      if (c < best) {
        best = c;
        plan.split = 1;
        plan.main_tiles = t1;
        plan.tail_split = S;
      }
    }
  }
  if (best > 0.98 * base) plan = DensePlan{1, tiles, 1};
  return plan;
}

template <int D>
int launch_cluster(const AttnArgs& a, cudaStream_t st, int S, int64_t tile0 = 0, int64_t ntiles = -1) {
  EncodeTiledFn enc;
  if (int e = tensor_map_encoder(&enc, "pruned_attn")) return e;
  int err;
  unsigned int* status = device_status(&err);
  if (!status) return err;
  CUtensorMap mq, mk, mv;
  if (int e = make_map(enc, &mq, a.q, a.cap, a.H, a.d)) return e;
  if (int e = make_map(enc, &mk, a.k, a.N, a.H, a.d)) return e;
  if (int e = make_map(enc, &mv, a.v, a.N, a.H, a.d)) return e;
  if (int e = smem_attribute<attn_tc_kernel<D, true>>(Layout<D, 1>::kAlloc)) return e;
  TcParams prm{a, a.scale * kLog2e, status, S, nullptr, nullptr, S, static_cast<int>(tile0)};
  if (ntiles < 0) ntiles = (a.cap + kQT * kBM - 1) / (kQT * kBM);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned int>(ntiles), static_cast<unsigned int>(a.H), static_cast<unsigned int>(S));
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Layout<D, 1>::kAlloc;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = static_cast<unsigned int>(S);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, attn_tc_kernel<D, true>, mq, mk, mv, prm);
  if (e != cudaSuccess) return cuda_status(e, "pruned_attn: cluster launch");
  return launch_status("pruned_attn");
}

// Key-range splits for a launch that would fill the GPU poorly: one pass of
// ceil(cap/256) x H CTAs that leaves most of its last wave empty (e.g. 156
// CTAs on 148 SMs) runs as S <= 4 key-range splits in one grid, followed by an
// S-way log-sum-exp merge. Dense mode only; >= 4 key tiles per split.
int choose_split(int64_t cap, int H, int64_t N, bool masked) {
  if (masked) return 1;
  const int64_t units = ((cap + kQT * kBM - 1) / (kQT * kBM)) * H;
  const int64_t sms = sm_count();
  const int64_t nkt = (N + kBN - 1) / kBN;
  auto eff = [&](int64_t s) {
    const int64_t u = units * s;
    return static_cast<double>(u) / static_cast<double>(((u + sms - 1) / sms) * sms);
  };
  if (units <= 0 || eff(1) >= 0.9) return 1;
  int best = 1;
  double be = eff(1);
  for (int s = 2; s <= 4; ++s) {
    if (nkt < 4 * s) break;
    const double e = eff(s);
    if (e > be + 0.02) {
      best = s;
      be = e;
    }
  }
  return best;
}

size_t split_ws_bytes(int nsplit, int64_t cap, int H, int d) {
  if (nsplit <= 1) return 0;
  const size_t o = static_cast<size_t>(nsplit) * cap * H * d * sizeof(float);
  return (o + 255) / 256 * 256 + static_cast<size_t>(nsplit) * cap * H * sizeof(float);
}

}  // namespace

// S-way merge of the split partials (merge.cu).
int merge_split_parts(const float* o_part, const float* lse_part, int nsplit, const int32_t* count, int64_t cap,
                      int H, int d, uint16_t* o, float* lse, cudaStream_t st);

}  // namespace tps

extern "C" size_t tps_attn_workspace_size(int64_t cap, int64_t N, int H, int d) {
  using namespace tps;
  if (cap <= 0 || N <= 0 || H <= 0 || (d != 64 && d != 128)) return 0;
  return split_ws_bytes(choose_split(cap, H, N, false), cap, H, d);
}

extern "C" int pruned_attn_ws(const tps_bf16* q_act, const tps_bf16* k, const tps_bf16* v, const int32_t* idx,
                              const int32_t* count, int64_t cap, int64_t N, int H, int d, float scale,
                              const uint8_t* blockmask, int block, tps_bf16* o_act, float* lse, void* ws,
                              size_t ws_bytes, tps_stream stream) {
  TPS_TRACE("pruned_attn_ws");
  using namespace tps;
  AttnArgs a;
  if (int e = attn_validate("pruned_attn_ws", q_act, k, v, idx, count, cap, N, H, d, scale, blockmask, block, o_act,
                            lse, &a))
    return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int S = choose_split(cap, H, N, blockmask != nullptr);
  const size_t need = split_ws_bytes(S, cap, H, d);
  if (S <= 1 || !ws || ws_bytes < need || !aligned16(ws)) {   // no split possible or needed
    const int e = d == 64 ? launch<64>(a, st) : launch<128>(a, st);
    return e ? e : ok();
  }
  float* o_part = static_cast<float*>(ws);
  float* lse_part = reinterpret_cast<float*>(static_cast<char*>(ws) +
                                             (static_cast<size_t>(S) * cap * H * d * sizeof(float) + 255) / 256 * 256);
  int e = d == 64 ? launch<64>(a, st, S, o_part, lse_part) : launch<128>(a, st, S, o_part, lse_part);
  if (e) return e;
  e = merge_split_parts(o_part, lse_part, S, count, cap, H, d, o_act, lse, st);
  return e ? e : ok();
}

// CTA-pair kernel for dense d = 128 launches (attn_pair.cu).
namespace tps {
int launch_pair(const AttnArgs& a, cudaStream_t st);
}

extern "C" int pruned_attn_pair(const tps_bf16* q_act, const tps_bf16* k, const tps_bf16* v, const int32_t* idx,
                                const int32_t* count, int64_t cap, int64_t N, int H, int d, float scale,
                                const uint8_t* blockmask, int block, tps_bf16* o_act, float* lse, tps_stream stream) {
  TPS_TRACE("pruned_attn_pair");
  using namespace tps;
  AttnArgs a;
  if (int e = attn_validate("pruned_attn_pair", q_act, k, v, idx, count, cap, N, H, d, scale, blockmask, block,
                            o_act, lse, &a))
    return e;
  if (d != 128 || blockmask)
    return fail(TPS_ERR_INVALID_ARG, "pruned_attn_pair: dense attention with d = 128 only (d=%d, mask %s)", d,
                blockmask ? "given" : "none");
  const int e = launch_pair(a, static_cast<cudaStream_t>(stream));
  return e ? e : ok();
}

extern "C" int tps_attn_split(int64_t cap, int64_t N, int H, int d) {
  using namespace tps;
  if (cap <= 0 || N <= 0 || H <= 0 || (d != 64 && d != 128)) return 1;
  return (d == 64 ? plan_dense<64>(cap, H, N) : plan_dense<128>(cap, H, N)).split;
}

extern "C" int tps_attn_plan(int64_t cap, int64_t N, int H, int d, int* split, int64_t* main_rows, int* tail_split) {
  using namespace tps;
  if (!split || !main_rows || !tail_split) return fail(TPS_ERR_INVALID_ARG, "tps_attn_plan: null pointer");
  if (cap < 0 || N <= 0 || H <= 0 || (d != 64 && d != 128))
    return fail(TPS_ERR_INVALID_ARG, "tps_attn_plan: need cap >= 0, N > 0, H > 0, d in {64, 128}");
  DensePlan plan;
  if (cap > 0) plan = d == 64 ? plan_dense<64>(cap, H, N) : plan_dense<128>(cap, H, N);
  *split = plan.split;
  *main_rows = plan.tail_split > 1 ? plan.main_tiles * (kQT * kBM) : cap;
  *tail_split = plan.tail_split;
  return ok();
}

extern "C" int pruned_attn(const tps_bf16* q_act, const tps_bf16* k, const tps_bf16* v, const int32_t* idx,
                           const int32_t* count, int64_t cap, int64_t N, int H, int d, float scale,
                           const uint8_t* blockmask, int block, tps_bf16* o_act, float* lse, tps_stream stream) {
  TPS_TRACE("pruned_attn");
  using namespace tps;
  AttnArgs a;
  if (int e = attn_validate("pruned_attn", q_act, k, v, idx, count, cap, N, H, d, scale, blockmask, block, o_act,
                            lse, &a))
    return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (blockmask || cap == 0) {
    const int e = d == 64 ? launch<64>(a, st) : launch<128>(a, st);
    return e ? e : ok();
  }
  const DensePlan plan = d == 64 ? plan_dense<64>(cap, H, N) : plan_dense<128>(cap, H, N);
  int e;
  if (plan.split > 1) {
    e = d == 64 ? launch_cluster<64>(a, st, plan.split) : launch_cluster<128>(a, st, plan.split);
  } else {
    e = d == 64 ? launch<64>(a, st, 1, nullptr, nullptr, 0, plan.main_tiles)
                : launch<128>(a, st, 1, nullptr, nullptr, 0, plan.main_tiles);
    const int64_t tiles = (cap + kQT * kBM - 1) / (kQT * kBM);
    if (!e && plan.tail_split > 1)
      e = d == 64 ? launch_cluster<64>(a, st, plan.tail_split, plan.main_tiles, tiles - plan.main_tiles)
                  : launch_cluster<128>(a, st, plan.tail_split, plan.main_tiles, tiles - plan.main_tiles);
  }
  return e ? e : ok();
}
