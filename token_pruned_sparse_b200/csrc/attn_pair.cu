// pruned_attn on CTA pairs: the dense path (d = 128) as one tcgen05 MMA of
// M = 256 over two SMs (cta_group::2), with the probabilities P in shared memory.
//
// [HSA] "Asignacion de Pasos Heterogenea", 2.2 (3)-(4): the active tokens'
// queries attend the full cached K/V, so the attention costs O(|A_i| * N).
//
// A cluster of two CTAs (ranks 0 and 1, one SM each) takes 512 compacted
// active queries of one head as two tiles t = 0, 1 of 256 rows; CTA c holds
// rows [256 t + 128 c, +128) of each tile. Per key tile of 128 keys:
//   S_t = Q_t K^T    M = 256 (each CTA's 128 query rows from its own shared
//                    memory), N = 128 keys (CTA c holds keys 64c..64c+63 of
//                    the tile), accumulated in each CTA's own TMEM;
//   O_t += P_t V     M = 256 (P_t: each CTA's 128 rows, bf16 in its shared
//                    memory), N = d = 128 (CTA c holds d columns 64c..64c+63
//                    of the 128 keys' V).
// Each SM thus reads half of every K and V tile from shared memory, and L2
// sends each SM half the K/V bytes. The shared memory that frees holds P, so
// S is released as soon as the softmax has read it: the next S = Q K^T runs
// on the tensor cores while the softmax of the current tile still works,
// instead of waiting for its P V.
//
// Warp roles in each CTA: warps 0-3 / 4-7 softmax of tile 0 / 1 (thread r owns
// row r of the CTA's half of the tile = TMEM lane r), warp 8 TMA producer
// (its own Q rows, its halves of K and V), warp 9 MMA issuer (rank 0 only;
// both ranks allocate the pair's TMEM). The softmax takes each tile's row
// maximum while S is in registers and then releases S, so the next Q K^T
// overlaps its exponentials (log2 domain, packed f32x2 arithmetic); the
// running reference maximum moves only when a tile's maximum exceeds it by
// more than 2^8, with the O accumulator rescaled in TMEM then. The MMA
// issuer runs both tiles' next Q K^T before their P V products.
//
// Synchronisation. Barriers that rank 1 also signals live in rank 0 and are
// waited on with acquire at cluster scope: TMA completions of both CTAs'
// loads (Q, K, V), "S read" and "P written" arrivals of both CTAs' softmax
// threads. MMA completions are committed to the barrier at the same offset in
// both CTAs (multicast commit): S ready, P V done, K and V stages free. Every
// wait is bounded (about 1 s); on expiry a CTA sets its abort flag and the
// device status word (TPS_ERR_TIMEOUT), drains what it issued and meets its
// peer at the final cluster barrier, which keeps both CTAs' shared memory and
// TMEM alive until neither has work in flight. TMA loads carry no multicast.
#include "trace.cuh"
#include "attn_common.cuh"
#include "tc_ptx.cuh"
#include "tma_host.cuh"

namespace tps {
namespace {

using namespace tc;

constexpr int kD = 128;
constexpr int kBM = 128;          // query rows per CTA per tile (half of M = 256)
constexpr int kQT = 2;            // tiles per pair
constexpr int kBN = 128;          // keys per tile
constexpr int kStages = 2;        // K / V ring depth
constexpr int kSoftmaxThreads = kQT * kBM;
constexpr int kThreads = kSoftmaxThreads + 64;
constexpr int kTmaWarp = kSoftmaxThreads / 32;
constexpr int kMmaWarp = kTmaWarp + 1;
constexpr int kTmemCols = 512;
constexpr int kRowsPerPair = 2 * kQT * kBM;      // 512 query rows per cluster
constexpr int kSub = 128 * 128;                  // [128 rows x 64 bf16], 128-byte swizzle
constexpr int kHalfSub = 64 * 128;               // [64 keys x 64 bf16] (a K half)
constexpr float kRefSlack = 8.f;                 // P < 2^8 between reference moves

struct PairLayout {
  static constexpr int kQ = 0;                                  // [tile][d half]  Q rows of this CTA
  static constexpr int kK = kQ + kQT * 2 * kSub;                // [stage][d half] 64 keys of the tile
  static constexpr int kV = kK + kStages * 2 * kHalfSub;        // [stage]         128 keys x 64 d
  static constexpr int kP = kV + kStages * kSub;                // [tile][key half] P rows of this CTA
  static constexpr int kBar = kP + kQT * 2 * kSub;
  static constexpr int kBytes = kBar + 256;
  static constexpr int kAlloc = kBytes + 1024;
};

struct PairBars {
  static constexpr int q_full = 0;                  // + tile   (rank 0: both CTAs' Q bytes)
  static constexpr int k_full = q_full + kQT;       // + stage  (rank 0: both halves)
  static constexpr int v_full = k_full + kStages;   // + stage  (rank 0: both halves)
  static constexpr int k_empty = v_full + kStages;  // + stage  (both: last S MMA of the stage)
  static constexpr int v_empty = k_empty + kStages; // + stage  (both: last P V MMA of the stage)
  static constexpr int s_full = v_empty + kStages;  // + tile   (both)
  static constexpr int pv_done = s_full + kQT;      // + tile   (both)
  static constexpr int s_read = pv_done + kQT;      // + tile   (rank 0: 256 softmax threads)
  static constexpr int p_full = s_read + kQT;       // + tile   (rank 0: 256 softmax threads)
  static constexpr int drain = p_full + kQT;        // rank 0: last commit
  static constexpr int count = drain + 1;
};
static_assert(PairBars::count * 8 <= 256, "barrier block");

struct PairParams {
  AttnArgs a;
  float scale_log2;
  unsigned int* status;
};

__global__ void __launch_bounds__(kThreads, 1)
attn_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKh,
                 const __grid_constant__ CUtensorMap tmVh, PairParams prm) {
  using L = PairLayout;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;

  const AttnArgs& p = prm.a;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  const uint32_t crank = cluster_ctarank();
  const bool lead = crank == 0;
  const int64_t rows = active_count(p.count, p.cap);
  const int64_t base = static_cast<int64_t>(blockIdx.x >> 1) * kRowsPerPair;
  if (base >= rows) return;                     // both CTAs of the pair leave together
  const int64_t row0 = base + crank * kBM;      // tile t: rows row0 + 256 t + [0, 128)

  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - smem_u32(smem_raw));
  const uint32_t bar0 = sbase + L::kBar;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  const uint32_t lbar0 = map_to_rank(bar0, 0);  // rank 0's barrier block, cluster address
  auto lbar = [&](int i) { return lbar0 + 8u * static_cast<uint32_t>(i); };
  const int ntiles = static_cast<int>((p.N + kBN - 1) / kBN);

  if (tid == 0) {
    s_abort = 0;
    for (int t = 0; t < kQT; ++t) {
      mbar_init(bar(PairBars::q_full + t), 1);
      mbar_init(bar(PairBars::s_full + t), 1);
      mbar_init(bar(PairBars::pv_done + t), 1);
      mbar_init(bar(PairBars::s_read + t), 2 * kBM);
      mbar_init(bar(PairBars::p_full + t), 2 * kBM);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(PairBars::k_full + s), 1);
      mbar_init(bar(PairBars::v_full + s), 1);
      mbar_init(bar(PairBars::k_empty + s), 1);
      mbar_init(bar(PairBars::v_empty + s), 1);
    }
    mbar_init(bar(PairBars::drain), 1);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tmem_alloc_pair<kTmemCols>(smem_u32(&s_tmem));
  if (warp == kTmaWarp && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmKh);
    tma_prefetch_desc(&tmVh);
  }
  tc_fence_before();
  __syncthreads();
  // both CTAs' barriers exist and the pair's TMEM is allocated before any
  // cross-CTA arrival, load completion or MMA
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  auto tS = [&](int t) { return tmem + 256u * t; };
  auto tO = [&](int t) { return tmem + 256u * t + 128u; };

  if (warp == kTmaWarp) {
    // ================================ TMA producer =====================================
    if (lane == 0) {
      constexpr uint32_t kQBytes = 2 * kSub, kKBytes = 2 * kHalfSub, kVBytes = kSub;   // per CTA
      int issued = 0;
      for (int t = 0; t < kQT; ++t) {
        if (lead) mbar_expect_tx(bar(PairBars::q_full + t), 2 * kQBytes);
        for (int s = 0; s < 2; ++s)
          tma_load_3d_pair(sbase + L::kQ + (t * 2 + s) * kSub, &tmQ, 64 * s, h, static_cast<int>(row0 + 2 * kBM * t),
                           lbar(PairBars::q_full + t));
      }
      for (int j = 0; j < ntiles; ++j) {
        const int st = j % kStages;
        const uint32_t ph = ((j / kStages) - 1) & 1;
        const int key0 = j * kBN;
        if (j >= kStages && !mbar_wait(bar(PairBars::k_empty + st), ph, &s_abort, prm.status)) break;
        if (lead) mbar_expect_tx(bar(PairBars::k_full + st), 2 * kKBytes);
        for (int s = 0; s < 2; ++s)
          tma_load_3d_pair(sbase + L::kK + (st * 2 + s) * kHalfSub, &tmKh, 64 * s, h, key0 + 64 * static_cast<int>(crank),
                           lbar(PairBars::k_full + st));
        if (j >= kStages && !mbar_wait(bar(PairBars::v_empty + st), ph, &s_abort, prm.status)) break;
        if (lead) mbar_expect_tx(bar(PairBars::v_full + st), 2 * kVBytes);
        tma_load_3d_pair(sbase + L::kV + st * kSub, &tmVh, 64 * static_cast<int>(crank), h, key0,
                         lbar(PairBars::v_full + st));
        issued = j + 1;
      }
      // drain (rank 0 counts both CTAs' bytes): every load must land before either CTA exits
      if (lead) {
        for (int t = 0; t < kQT; ++t) drain_wait(bar(PairBars::q_full + t), 0);
        for (int j = issued > kStages ? issued - kStages : 0; j < issued; ++j) {
          drain_wait(bar(PairBars::k_full + j % kStages), (j / kStages) & 1);
          drain_wait(bar(PairBars::v_full + j % kStages), (j / kStages) & 1);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ================================ MMA issuer (rank 0) ==============================
    if (lead && lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16(2 * kBM, kBN, false, false);   // Q K^T, both K-major
      constexpr uint32_t kIdescO = idesc_bf16(2 * kBM, kD, false, true);     // P V, V MN-major
      constexpr uint16_t kBoth = 0x3;
      auto issue_s = [&](int t, int j) {
        const int st = j % kStages;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t da = sdesc_sw128(sbase + L::kQ + (t * 2 + (kk >> 2)) * kSub + (kk & 3) * 32, 16, 1024);
          const uint64_t db = sdesc_sw128(sbase + L::kK + (st * 2 + (kk >> 2)) * kHalfSub + (kk & 3) * 32, 16, 1024);
          mma_f16_ss_pair(tS(t), da, db, kIdescS, kk > 0);
        }
        mma_commit_pair(bar(PairBars::s_full + t), kBoth);
        if (t == kQT - 1) mma_commit_pair(bar(PairBars::k_empty + st), kBoth);
      };
      auto issue_pv = [&](int t, int j) {
        const int st = j % kStages;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          // A = P_t, K-major over keys: 16 keys per step, 64 keys per swizzled half.
          // B = V half, MN-major: 16 keys = 2 swizzle atoms of 8 keys.
          const uint64_t da = sdesc_sw128(sbase + L::kP + (t * 2 + (kk >> 2)) * kSub + (kk & 3) * 32, 16, 1024);
          const uint64_t db = sdesc_sw128(sbase + L::kV + st * kSub + kk * 16 * 128, kSub, 1024);
          mma_f16_ss_pair(tO(t), da, db, kIdescO, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit_pair(bar(PairBars::pv_done + t), kBoth);
        if (t == kQT - 1) mma_commit_pair(bar(PairBars::v_empty + st), kBoth);
      };
      bool ok = ntiles > 0 && mbar_wait_cluster(bar(PairBars::k_full), 0, &s_abort, prm.status);
      for (int t = 0; ok && t < kQT; ++t) {
        ok = mbar_wait_cluster(bar(PairBars::q_full + t), 0, &s_abort, prm.status);
        tc_fence_after();
        if (ok) issue_s(t, 0);
      }
      for (int j = 0; ok && j < ntiles; ++j) {
        // S of the next key tile for both tiles first: each is released as soon as
        // the softmax has S in registers, long before its P is ready
        for (int t = 0; ok && t < kQT && j + 1 < ntiles; ++t) {
          // the softmax of both CTAs has read S_t(j): S_t(j+1) may overwrite it
          ok = mbar_wait_cluster(bar(PairBars::s_read + t), j & 1, &s_abort, prm.status);
          if (ok && t == 0)
            ok = mbar_wait_cluster(bar(PairBars::k_full + (j + 1) % kStages), ((j + 1) / kStages) & 1, &s_abort,
                                   prm.status);
          tc_fence_after();
          if (ok) issue_s(t, j + 1);
        }
        for (int t = 0; ok && t < kQT; ++t) {
          ok = mbar_wait_cluster(bar(PairBars::p_full + t), j & 1, &s_abort, prm.status);
          if (ok && t == 0)
            ok = mbar_wait_cluster(bar(PairBars::v_full + j % kStages), (j / kStages) & 1, &s_abort, prm.status);
          tc_fence_after();
          if (ok) issue_pv(t, j);
        }
      }
      mma_commit_pair(bar(PairBars::drain), 0x1);   // fires once every MMA issued above has completed
    }
  } else {
    // ================================ softmax warps ====================================
    const int t = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const int64_t row = row0 + 2 * kBM * t + r;
    const bool valid = row < rows;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_read_bar = lead ? bar(PairBars::s_read + t) : lbar(PairBars::s_read + t);
    const uint32_t p_full_bar = lead ? bar(PairBars::p_full + t) : lbar(PairBars::p_full + t);
    // this thread's row of P_t: two 64-key halves, 128 bytes per row, 16-byte chunks XOR-swizzled by row
    uint8_t* prow = gbase + L::kP + t * 2 * kSub + r * 128;
    const int sw = r & 7;
    const float sl2 = prm.scale_log2;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar(PairBars::s_full + t), j & 1, &s_abort, prm.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int64_t key0 = static_cast<int64_t>(j) * kBN;
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
      auto exp_pass = [&](float base_m) -> float {
        const uint64_t nbase = f2_pack(-base_m, -base_m);
        uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = acc0;
#pragma unroll
        for (int c = 0; c < kBN; c += 4) {
          float a0, a1, a2, a3;
          f2_unpack(ffma2(f2_pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl2x2, nbase), a0, a1);
          f2_unpack(ffma2(f2_pack(__uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3])), sl2x2, nbase), a2, a3);
          const float p0 = fast_exp2(a0), p1 = fast_exp2(a1), p2 = fast_exp2(a2), p3 = fast_exp2(a3);
          acc0 = fadd2(acc0, f2_pack(p0, p1));
          acc1 = fadd2(acc1, f2_pack(p2, p3));
          pk[c >> 1] = pack_bf16x2(p0, p1);
          pk[(c >> 1) + 1] = pack_bf16x2(p2, p3);
        }
        float s0, s1, s2, s3;
        f2_unpack(acc0, s0, s1);
        f2_unpack(acc1, s2, s3);
        return (s0 + s1) + (s2 + s3);
      };
      load_s();
      // The row maximum of every tile is taken while S is in registers, so S
      // can be released at once: the next Q K^T then overlaps this tile's
      // exponentials. The reference maximum moves only when the tile's
      // maximum exceeds it by more than kRefSlack (log2 units), which keeps
      // every P below 2^kRefSlack and makes O rescales rare.
      float mx0 = __uint_as_float(sr[0]), mx1 = __uint_as_float(sr[1]);
      float mx2 = __uint_as_float(sr[2]), mx3 = __uint_as_float(sr[3]);
#pragma unroll
      for (int c = 4; c < kBN; c += 4) {
        mx0 = fmaxf(mx0, __uint_as_float(sr[c]));
        mx1 = fmaxf(mx1, __uint_as_float(sr[c + 1]));
        mx2 = fmaxf(mx2, __uint_as_float(sr[c + 2]));
        mx3 = fmaxf(mx3, __uint_as_float(sr[c + 3]));
      }
      // S_t(j) is in registers: the next Q K^T may overwrite it
      tc_fence_before();
      if (lead) mbar_arrive(s_read_bar);
      else mbar_arrive_remote(s_read_bar);
      const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
      const float m_target = m_run == -INFINITY || m_tile > m_run + kRefSlack ? fmaxf(m_run, m_tile) : m_run;
      if (j > 0 && __any_sync(0xffffffffu, m_target > m_run)) {
        // O (complete up to tile j-1) moves to the new reference
        const float alpha = m_run == -INFINITY ? 0.f : fast_exp2(m_run - m_target);
        if (!__all_sync(0xffffffffu, mbar_wait(bar(PairBars::pv_done + t), (j - 1) & 1, &s_abort, prm.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < kD; c += 32) {
          float o[32];
          tmem_ld32(tO(t) + lane_off + c, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(tO(t) + lane_off + c, o);
        }
        l_run *= alpha;
      }
      m_run = m_target;
      l_run += exp_pass(m_run == -INFINITY ? 0.f : m_run);
      // P_t(j-1) must have been consumed before its buffer is overwritten
      if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(bar(PairBars::pv_done + t), (j - 1) & 1, &s_abort, prm.status))) {
        ok = false;
        break;
      }
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int k = hf * 32 + c * 4;
          *reinterpret_cast<uint4*>(prow + hf * kSub + ((c ^ sw) << 4)) = make_uint4(pk[k], pk[k + 1], pk[k + 2], pk[k + 3]);
        }
      fence_proxy_async_smem();                  // generic-proxy P writes -> the MMA's async-proxy reads
      if (lead) mbar_arrive(p_full_bar);
      else mbar_arrive_remote(p_full_bar);
    }
    // ---- epilogue ------------------------------------------------------------------------
    if (ok && ntiles > 0) ok = mbar_wait(bar(PairBars::pv_done + t), (ntiles - 1) & 1, &s_abort, prm.status);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    if (ok) {
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      uint4* orow = reinterpret_cast<uint4*>(p.o + (row * p.H + h) * kD);
#pragma unroll
      for (int c = 0; c < kD; c += 32) {
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

  // ---- teardown ------------------------------------------------------------------------
  if (lead && warp == kMmaWarp && lane == 0) drain_wait(bar(PairBars::drain), 0);
  tc_fence_before();
  __syncthreads();
  // neither CTA frees TMEM or leaves while the pair's MMAs or loads may touch it
  cluster_sync_all();
  tc_fence_after();
  if (warp == kMmaWarp) {
    __syncwarp();
    tmem_dealloc_pair<kTmemCols>(tmem);
  }
}

// [rows, H, d] bf16 -> 3-D map (d, H, rows), box (64, 1, box_rows), 128-byte swizzle.
int make_pair_map(EncodeTiledFn enc, CUtensorMap* m, const void* ptr, int64_t rows, int H, int d, int box_rows) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H) * d * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TPS_ERR_CUDA, "pruned_attn: cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return TPS_OK;
}

}  // namespace

// Pairs of CTAs resident at once (cudaOccupancyMaxActiveClusters for clusters
// of two), cached per device; 0 if the pair kernel cannot be scheduled.
int pair_slots() {
  static std::atomic<int> cache[64];   // slots + 1; 0 = not yet queried
  int dev = 0;
  cudaGetDevice(&dev);
  const bool cacheable = dev >= 0 && dev < 64;
  if (cacheable) {
    const int v = cache[dev].load(std::memory_order_acquire);
    if (v > 0) return v - 1;
  }
  int n = 0;
  if (cudaFuncSetAttribute(attn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PairLayout::kAlloc) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = PairLayout::kAlloc;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, attn_pair_kernel, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();                 // a failed query leaves its error in the last-error slot
  if (cacheable) cache[dev].store(n + 1, std::memory_order_release);
  return n;
}

// Dense pruned_attn of d = 128 on CTA pairs: ceil(cap/512) x H clusters of two.
int launch_pair(const AttnArgs& a, cudaStream_t st) {
  if (a.cap == 0) return TPS_OK;
  EncodeTiledFn enc;
  if (int e = tensor_map_encoder(&enc, "pruned_attn")) return e;
  int err;
  unsigned int* status = device_status(&err);
  if (!status) return err;
  CUtensorMap mq, mk, mv;
  if (int e = make_pair_map(enc, &mq, a.q, a.cap, a.H, a.d, 128)) return e;
  if (int e = make_pair_map(enc, &mk, a.k, a.N, a.H, a.d, 64)) return e;
  if (int e = make_pair_map(enc, &mv, a.v, a.N, a.H, a.d, 128)) return e;
  if (pair_slots() <= 0) return fail(TPS_ERR_CUDA, "pruned_attn: CTA pairs cannot be scheduled on this device");
  PairParams prm{a, a.scale * kLog2e, status};
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned int>(2 * ((a.cap + kRowsPerPair - 1) / kRowsPerPair)),
                     static_cast<unsigned int>(a.H), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = PairLayout::kAlloc;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, attn_pair_kernel, mq, mk, mv, prm);
  if (e != cudaSuccess) return cuda_status(e, "pruned_attn: pair launch");
  return launch_status("pruned_attn");
}

}  // namespace tps
