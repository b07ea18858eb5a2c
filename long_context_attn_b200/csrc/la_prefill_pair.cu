// Lightning Attention prefill on the 5th-generation tensor cores, one head per CTA pair
// with the sequence split between the two CTAs block by block.
//
// What is computed ("六十四：MiniMax-01", section 3; "MiniMax-Text-01 405B MoE模型架构与
// 训练策略解析", section 2.1; "MiniMax-01技术报告解读（二）计算优化", section 3): causal
// linear attention with phi = SiLU on q and k, evaluated block by block with the block
// size C (256 in the deployment config).  For block j with rows Q_j, K_j, V_j:
//     O_j = (phi(Q_j) phi(K_j)^T (.) M) V_j + phi(Q_j) S_{j-1}          (intra + inter)
//     S_j = S_{j-1} + phi(K_j)^T V_j                                    (fp32 state carry)
// followed by o = RMSNorm over the H*D head concatenation of a token times sigmoid(g).
//
// Design (B200, sm_100a):
//  * The two CTAs of a cluster work on one head; each is a worker that owns whole sequences
//    (a long sequence arrives cut into chunks, each with its initial state, from the host
//    side) and carries their state in its own TMEM, so no state crosses between SMs.  With
//    G sequence groups there are 2G workers per head; a worker's sequences come from a plan
//    (longest first over the workers) or round robin.  Every worker processes full head
//    width: every MMA is 128 x 128 (N = 128) and each score is computed once per head.
//  * Tiles are 128 rows (the MMA M).  C = 256 is two tiles per block: tile 1 multiplies by
//    tile 0's keys densely and by its own keys under the causal mask.  Tails use N / K
//    extents of 32, 64 or 128 rows (`lightning_attention_pad_options`) with zeroed tail rows
//    of K and V.  The inter product phi(Q_b) S_{b-1} uses a bf16 snapshot of the state that
//    the state warps take after the previous block's last state update.
//  * Roles (32 warps): warp 0 streams Q, K and V tiles with TMA into two-slot rings (one
//    lane per ring); warp 1 issues every MMA; warps 2, 3 and 24-31 apply SiLU (packed
//    bf16x2 arithmetic) to K in place; warps 4-7 turn score tiles into masked bf16 in TMEM;
//    warps 8-11 apply SiLU to Q on its way into TMEM; warps 12-15 own the state (S0 in, the
//    snapshot, the final state out) and the output accumulator (each row read once,
//    written out and, in the norm modes, its sum of squares published); warps 16-23, once
//    all heads of a tile have published, rescale its rows in place:
//    o = z rsqrt(mean(y^2) + eps) sigmoid(g) with z = bf16(y w).
//  * TMEM (512 columns): S (128), the output accumulator (128), one score region (128),
//    phi(Q) of two tiles (2 x 64, the A operand of the score and inter MMAs).  The three
//    score jobs of a block go through the one region back to back: MMAs of one thread run
//    in issue order, so each job is issued right after the previous job's PV.
//  * Cross-head RMSNorm: every drain thread adds its row's sum of squares into an fp64
//    per-token total (red.add; exact and order-independent while a token's partials span
//    less than 2^22), and each warp bumps the tile's arrival counter after a fence.  The
//    same worker of every head processes the same tiles in the same order, and all CTAs are
//    resident at once (checked on the host).  A CTA's Q loads wait until every head has
//    published the tile kThrottle tiles back, so the rows waiting for their rescale stay
//    few enough to remain in L2.
//  * Every wait is bounded (globaltimer); a wait that runs out records LA_ERR_TIMEOUT in
//    the workspace, raises the CTA's abort flag and the CTA drains its async work, frees
//    TMEM and exits.
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <mutex>

#include "la_common.cuh"
#include "la_prefill_tc.h"
#include "la_sm100.cuh"
#include "la_tc_util.cuh"

namespace la {
using namespace sm100;
using tcu::lds128;
using tcu::sts128;

namespace {

constexpr int kD = 128;           // head dim (d_k = d_v)
constexpr int kTile = 128;        // rows per tile (MMA M)
constexpr int kThreads = 1024;    // 32 warps
constexpr int kConvWarp0 = 4;     // warps 4..7: score conversion
constexpr int kQxfWarp0 = 8;      // warps 8..11: SiLU of Q into TMEM (one TMEM lane quarter each)
constexpr int kStateWarp0 = 12;   // warps 12..15: the state and the rows' sums of squares
constexpr int kXfThreads = 320;   // warps 2, 3, 24..31: SiLU of K in place
constexpr int kXfIlp = 4;         // 16-byte chunks in flight per K-transform thread
constexpr int kEpiWarp0 = 16;     // warps 16..23: the normalised output (norm modes)
constexpr int kEpiWarps = 8;
constexpr int kXfWarp1 = 24;      // first of the K-transform warps after the output warps
constexpr int kPubWarps = 4;      // arrivals per CTA that publish a tile's sums
// Norm modes: the Q loads of own tile t wait until every head has published the sums of own
// tile t - kThrottle, so that no CTA runs far ahead of the slowest head.  The rows each CTA
// has written but not yet rescaled then stay few enough to remain in L2 until the final
// warps read them back.
constexpr int kThrottle = 6;

constexpr uint32_t kBoxBytes = kTile * 64 * 2;    // one 128-row x 64-column bf16 box (16 KiB)
constexpr uint32_t kTileBytes = 2 * kBoxBytes;    // a 128 x 128 tile: two boxes (32 KiB)
constexpr uint32_t OFF_Q = 0;                     // 2 slots (landing only: phi(Q) moves to TMEM)
constexpr uint32_t OFF_K = OFF_Q + 2 * kTileBytes;   // 2 slots
constexpr uint32_t OFF_V = OFF_K + 2 * kTileBytes;
constexpr uint32_t OFF_SNAP = OFF_V + 2 * kTileBytes;
constexpr uint32_t OFF_BARS = OFF_SNAP + kTileBytes;

// Norm exchange in global memory: one 128-byte line per token sum and per tile counter, so
// that the 64 heads' additions to one tile's sums spread over many L2 slices instead of
// queueing on the eight lines 128 packed fp64 values would share.
constexpr int kSsStride = 16;    // doubles per token
constexpr int kCntStride = 32;   // counters per tile

constexpr uint32_t TM_S = 0;      // S, 128 columns (lanes = d_k, columns = d_v)
constexpr uint32_t TM_O = 128;    // the output accumulator, 128 columns
constexpr uint32_t TM_P = 256;    // the score region, 128 columns
constexpr uint32_t TM_Q = 384;    // phi(Q) of two tiles, 64 columns each (bf16 pairs; MMA A operand)
constexpr uint32_t kTmemCols = 512;

struct Bars {
  uint64_t full_q[2], q_empty[2];      // Q landing slots (freed once phi(Q) is in TMEM)
  uint64_t qt_ready[2], qt_free[2];    // phi(Q) tiles in TMEM
  uint64_t full_k[2], xf_k[2], k_empty[2];
  uint64_t full_v[2], v_empty[2];
  uint64_t p_full, p_conv;
  uint64_t o_full, o_empty;
  uint64_t s_ready;     // S in TMEM may take the block's state update (S0 written / S_{b-1} read)
  uint64_t snap_ready;  // bf16 snapshot of S_{b-1} written
  uint64_t su_done;     // the block's state update (and its inter products) completed
  uint64_t final_bar;
  uint32_t tmem_base;
  int abort_flag;
  float w[kD];
};
constexpr uint32_t kSmemBytes = OFF_BARS + sizeof(Bars) + 1024;   // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct PairParams {
  const float* state_in;
  float* state_out;
  const int* cu;
  int nseq, T, H, phi_identity, max_tiles, ngroups;
  int chunk_div;            // > 1: sequences are chunks of chunk_div; only a last chunk writes state_out
  int64_t tokens;
  float eps;
  const float* w;
  const uint16_t* g;        // gate [tokens, H * D] (gated mode)
  ErrRec* err;
  unsigned int* cnt;        // [nseq * max_tiles] arrivals per tile
  double* ss;               // [tokens] sum of squares over the head concatenation
  const int* sched;         // optional [nseq]: sequences ordered by worker
  const int* wstart;        // optional [2 * ngroups + 1]: first entry of each worker in sched
  uint16_t* out;
  const int* state_index;   // optional [nseq]: state slot of each sequence (else the index)
  int skip_single;          // nonzero: one-token sequences belong to a decode step: skip them
};

constexpr uint64_t sdesc_template(uint32_t lbo, uint32_t sbo) {
  return (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) | (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) |
         (1ull << 46) | (2ull << 61);
}
constexpr uint64_t kDescK = sdesc_template(16, 1024);          // K-major, 128-byte swizzle
constexpr uint64_t kDescMN = sdesc_template(kBoxBytes, 1024);  // MN-major, 64-element chunks a box apart
// Descriptor of the operand at shared address `a` (14-bit start field: only the low 18
// address bits enter, so the cluster rank bits of a shared::cluster address never spill).
__device__ __forceinline__ uint64_t desc_at(uint64_t tmpl, uint32_t a) { return tmpl + ((a >> 4) & 0x3FFFu); }
// K-step kk (16 elements of K) of a K-major tile held as two 64-column boxes.
__device__ __forceinline__ uint64_t kstep_k(int kk) {
  return static_cast<uint64_t>(((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4);
}

constexpr uint32_t kIdesc128MN = make_idesc_bf16(128, 128, 0, 1);   // PV, QS: B MN-major
constexpr uint32_t kIdescSU = make_idesc_bf16(128, 128, 1, 1);      // S update: A and B MN-major

__device__ __forceinline__ int pad_rows(int vr) { return vr <= 32 ? 32 : (vr <= 64 ? 64 : 128); }

// Rows [row0, row0 + L) of sequence s (varlen checks as the other tensor-core kernel).
// Returns true for a one-token sequence of a mixed step (left alone entirely).
__device__ __forceinline__ bool seq_range(const PairParams& p, int s, int64_t& row0, int& L) {
  if (p.cu) {
    const int a = __ldg(p.cu + s), b = __ldg(p.cu + s + 1);
    row0 = a;
    L = b - a;
    if (a < 0 || L < 0 || static_cast<int64_t>(b) > p.tokens || ((L + kTile - 1) / kTile) > p.max_tiles) {
      if (threadIdx.x == 0) report(p.err, LA_ERR_DEVICE, SITE_VARLEN_CU, s, 0);
      L = 0;
    }
    if (p.skip_single && L == 1) {
      L = 0;
      return true;
    }
  } else {
    row0 = static_cast<int64_t>(s) * p.T;
    L = p.T;
  }
  return false;
}

// The blocks this worker walks: its sequences (from the plan, or every 2G-th) in order,
// each cut into blocks of tpb tiles; k indexes the worker's sequence list.
struct BlkIter {
  int k, kend, s, L, nt, jb, nblk;
  int64_t row0;
  bool valid;
};
__device__ __forceinline__ int worker_seq(const PairParams& p, int w, int k) {
  return p.sched ? __ldg(p.sched + k) : w + k * 2 * p.ngroups;
}
template <int tpb>
__device__ __forceinline__ void blk_seek(const PairParams& p, BlkIter& it, int w) {
  for (; it.k < it.kend; ++it.k) {
    const int s = worker_seq(p, w, it.k);
    int64_t r0;
    int L;
    seq_range(p, s, r0, L);
    const int nt = (L + kTile - 1) / kTile;
    if (nt > 0) {
      it.s = s;
      it.L = L;
      it.nt = nt;
      it.jb = 0;
      it.nblk = (nt + tpb - 1) / tpb;
      it.row0 = r0;
      it.valid = true;
      return;
    }
  }
  it.valid = false;
}
__device__ __forceinline__ void worker_range(const PairParams& p, int w, int& k0, int& k1) {
  if (p.sched) {
    k0 = __ldg(p.wstart + w);
    k1 = __ldg(p.wstart + w + 1);
  } else {
    const int nw = 2 * p.ngroups;
    k0 = 0;
    k1 = w < p.nseq ? (p.nseq - w + nw - 1) / nw : 0;
  }
}
template <int tpb>
__device__ __forceinline__ void blk_first(const PairParams& p, BlkIter& it, int w) {
  worker_range(p, w, it.k, it.kend);
  blk_seek<tpb>(p, it, w);
}
template <int tpb>
__device__ __forceinline__ void blk_next(const PairParams& p, BlkIter& it, int w) {
  if (it.jb + 1 < it.nblk) {
    ++it.jb;
    return;
  }
  ++it.k;
  blk_seek<tpb>(p, it, w);
}
// The tile of a sequence that walk position i covers: time forwards walks tiles 0 .. nt - 1,
// time backwards nt - 1 .. 0 (rows keep their order inside a tile).
template <bool rev>
__device__ __forceinline__ int phys_tile(int i, int nt) {
  return rev ? nt - 1 - i : i;
}
// Tiles of the current block and the valid rows of each.
template <int tpb, bool rev>
__device__ __forceinline__ int blk_tiles(const BlkIter& it, int& vr0, int& vr1) {
  const int t0 = it.jb * tpb;
  const int n = min(tpb, it.nt - t0);
  vr0 = min(kTile, it.L - phys_tile<rev>(t0, it.nt) * kTile);
  vr1 = n > 1 ? min(kTile, it.L - phys_tile<rev>(t0 + 1, it.nt) * kTile) : 0;
  return n;
}

// One 128 x 128 bf16 tile (two swizzled boxes) in place: SiLU on rows < zero_from, zero
// on the rest (phi = identity only zeroes).  All of a thread's 16-byte chunks are loaded
// before any is written back (up to kXfIlp in flight), so the MUFU stays busy.
__device__ __forceinline__ void xf_tile(uint32_t base, int zero_from, bool silu, int wt) {
  constexpr int kChunks = static_cast<int>(kTileBytes / 16);   // 2048
  for (int c0 = wt; c0 < kChunks; c0 += kXfIlp * kXfThreads) {
    uint4 v[kXfIlp];
#pragma unroll
    for (int j = 0; j < kXfIlp; ++j) {
      const int c = c0 + j * kXfThreads;
      v[j] = (c < kChunks) ? lds128(base + 16u * c) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < kXfIlp; ++j) {
      const int c = c0 + j * kXfThreads;
      if (c < kChunks) {
        const int row = (c & 1023) >> 3;   // 8 chunks of 16 bytes per 128-byte row of a box
        uint4 x = v[j];
        if (row >= zero_from) x = make_uint4(0, 0, 0, 0);
        else if (silu) x = tcu::silu8(x);
        sts128(base + 16u * c, x);
      }
    }
  }
}
// Zero rows >= vr of a 128 x 128 tile (the value tile of a sequence's last tile).
__device__ __forceinline__ void zero_tail(uint32_t base, int vr, int wt) {
  constexpr int kChunks = static_cast<int>(kTileBytes / 16);
  for (int c = wt; c < kChunks; c += kXfThreads)
    if (((c & 1023) >> 3) >= vr) sts128(base + 16u * c, make_uint4(0, 0, 0, 0));
}

// ======================================================================================
// The kernel (one instantiation per output mode and block size)
// ======================================================================================
template <int kMode, int kC, bool kRev>
__global__ void __launch_bounds__(kThreads, 1)
lightning_prefill_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                              const PairParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw_addr);
  Bars& B = *reinterpret_cast<Bars*>(smem + OFF_BARS);

  constexpr int tpb = kC / kTile;
  constexpr bool norm = kMode != LA_OUT_RAW;
  constexpr bool gate = kMode == LA_OUT_RMSNORM_GATE;
  static_assert(!kRev || kMode == LA_OUT_RAW, "time runs backwards in the raw mode only");
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int rank = static_cast<int>(cluster_ctarank());   // == blockIdx.x % 2
  const int pair = blockIdx.x >> 1;
  const int h = pair % p.H;
  const int wk = 2 * (pair / p.H) + rank;                  // worker: group * 2 + rank
  const uint32_t W = static_cast<uint32_t>(p.H * kPubWarps);   // arrivals that complete a tile's norm
  int* abort_flag = &B.abort_flag;
  ErrRec* err = p.err;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&B.qt_ready[i], 4);
      mbar_init(&B.qt_free[i], 1);
      mbar_init(&B.full_q[i], 1);
      mbar_init(&B.q_empty[i], 4);   // the Q-transform warps
      mbar_init(&B.full_k[i], 1);
      mbar_init(&B.xf_k[i], kXfThreads);
      mbar_init(&B.k_empty[i], 1);
      mbar_init(&B.full_v[i], 1);
      mbar_init(&B.v_empty[i], 1);
    }
    mbar_init(&B.p_full, 1);
    mbar_init(&B.p_conv, 128);
    mbar_init(&B.o_full, 1);
    mbar_init(&B.o_empty, 4);   // the four drain warps
    mbar_init(&B.s_ready, 128);
    mbar_init(&B.snap_ready, 128);
    mbar_init(&B.su_done, 1);
    mbar_init(&B.final_bar, 1);
    B.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc<kTmemCols>(&B.tmem_base);
  if (tid >= 32 * kEpiWarp0 && tid < 32 * kEpiWarp0 + kD) {
    const int c = tid - 32 * kEpiWarp0;
    B.w[c] = p.w ? p.w[h * kD + c] : 1.0f;
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = B.tmem_base;

  // ------------------------------------------------------------------------------------
  // Warp 0: TMA producers, one lane per two-slot ring: lane 0 Q tiles, lane 1 K tiles (and
  // the gate tile prefetched into L2 for the output), lane 2 V tiles.  Own tiles are numbered
  // in walk order and every ring uses that number: tile t goes to slot t % 2.  Each tile of
  // the next block is also prefetched into L2 when its load is issued.
  // ------------------------------------------------------------------------------------
  if (warp == 0) {
    if (lane < 3) {
      const CUtensorMap* map = lane == 0 ? &tm_q : (lane == 1 ? &tm_k : &tm_v);
      prefetch_tmap(map);
      if (lane == 1 && gate) prefetch_tmap(&tm_g);
      uint64_t* full = lane == 0 ? B.full_q : (lane == 1 ? B.full_k : B.full_v);
      uint64_t* empty = lane == 0 ? B.q_empty : (lane == 1 ? B.k_empty : B.v_empty);
      const uint32_t off = lane == 0 ? OFF_Q : (lane == 1 ? OFF_K : OFF_V);
      constexpr uint32_t sh = 1;   // log2 of the slots per ring
      const uint64_t pol = policy_evict_first();
      uint32_t ot = 0;
      bool ok = true;
      unsigned int* hist[kThrottle];   // norm counters of the last kThrottle own tiles (Q lane)
#pragma unroll
      for (int j = 0; j < kThrottle; ++j) hist[j] = nullptr;
      BlkIter it;
      blk_first<tpb>(p, it, wk);
      for (; it.valid && ok; blk_next<tpb>(p, it, wk)) {
        int vr0, vr1;
        const int n = blk_tiles<tpb, kRev>(it, vr0, vr1);
        for (int u = 0; u < n; ++u, ++ot) {
          if (norm && lane == 0) {
            unsigned int* c = hist[kThrottle - 1];
            if (c && ld_acquire_gpu(c) < W && !tcu::poll_count(c, W, abort_flag, err, ot)) {
              ok = false;
              break;
            }
#pragma unroll
            for (int j = kThrottle - 1; j > 0; --j) hist[j] = hist[j - 1];
            hist[0] = p.cnt + (static_cast<int64_t>(it.s) * p.max_tiles + it.jb * tpb + u) * kCntStride;
          }
          const uint32_t sl = ot & sh, use = ot >> sh;   // slot, and the loads into it before
          if (use >= 1 && !tcu::wait(&empty[sl], (use - 1) & 1u, abort_flag, err, SITE_TC_PRODUCER, ot)) {
            ok = false;
            break;
          }
          const int wi = it.jb * tpb + u;   // walk position of the tile
          const int32_t row = static_cast<int32_t>(it.row0 + static_cast<int64_t>(phys_tile<kRev>(wi, it.nt)) * kTile);
          const int32_t col = h * kD;
          if (wi + tpb < it.nt) {   // the same tile of the next block
            const int32_t nrow =
                static_cast<int32_t>(it.row0 + static_cast<int64_t>(phys_tile<kRev>(wi + tpb, it.nt)) * kTile);
            tma_prefetch_l2_2d(map, col, nrow);
            tma_prefetch_l2_2d(map, col + 64, nrow);
          }
          uint8_t* dst = smem + off + sl * kTileBytes;
          mbar_arrive_expect_tx(&full[sl], kTileBytes);
          tma_load_2d(dst, map, col, row, &full[sl], pol);
          tma_load_2d(dst + kBoxBytes, map, col + 64, row, &full[sl], pol);
          if (lane == 1 && gate) {
            tma_prefetch_l2_2d(&tm_g, col, row);
            tma_prefetch_l2_2d(&tm_g, col + 64, row);
          }
        }
      }
      // Drain: every issued load must land before the CTA may exit (the last load into
      // each slot is own tile ot - 1, or ot - 2 for the other slot of a two-slot ring).
      for (uint32_t sl = 0; sl <= sh; ++sl) {
        if (ot <= sl) continue;
        const uint32_t t = ((ot - 1) & sh) == sl ? ot - 1 : ot - 2;
        tcu::drain(&full[sl], (t >> sh) & 1u);
      }
    }
  }
  // ------------------------------------------------------------------------------------
  // Warp 1: MMA issuer (one thread).
  // ------------------------------------------------------------------------------------
  else if (warp == 1) {
    if (lane == 0) {
      uint32_t ot = 0, nb = 0, jb = 0;
      bool ok = true;
      BlkIter it;
      blk_first<tpb>(p, it, wk);
      auto mw = [&](uint64_t* bar, uint32_t par, uint32_t idx) -> bool {
        if (!tcu::wait(bar, par, abort_flag, err, SITE_TC_MMA, idx)) return false;
        tc_fence_after();
        return true;
      };
      // Score job phi(Q) K^T (A = phi(Q) of Q tile qs in TMEM) into the score region.  MMAs
      // issued by one thread execute in issue order, so the job may follow the previous job's
      // PV (which reads the converted scores there) without waiting for it to complete.
      auto issue_p = [&](uint32_t qs, uint32_t ks, uint32_t n) {
        const uint64_t kd = desc_at(kDescK, sbase + OFF_K + ks * kTileBytes);
        const uint32_t idesc = make_idesc_bf16(128, n, 0, 0);
#pragma unroll 1
        for (int kk = 0; kk < 8; ++kk) mma_ts(tmem + TM_P, tmem + TM_Q + 64 * qs + 8 * kk, kd + kstep_k(kk), idesc, kk > 0);
        mma_commit(&B.p_full);
      };
      // PV of the converted scores into the accumulator over ksteps key steps.
      auto issue_pv = [&](uint32_t vs, int ksteps, bool acc) -> bool {
        if (!mw(&B.p_conv, jb & 1u, jb)) return false;
        const uint64_t vd = desc_at(kDescMN, sbase + OFF_V + vs * kTileBytes);
#pragma unroll 1
        for (int kk = 0; kk < ksteps; ++kk)
          mma_ts(tmem + TM_O, tmem + TM_P + 8 * kk, vd + 128 * kk, kIdesc128MN, (acc || kk > 0) ? 1u : 0u);
        ++jb;
        return true;
      };
      // S += phi(K)^T V over the keys of one tile (S was set by the state warps).
      auto issue_su = [&](uint32_t ks, int ksteps) {
        const uint64_t kd = desc_at(kDescMN, sbase + OFF_K + ks * kTileBytes);
        const uint64_t vd = desc_at(kDescMN, sbase + OFF_V + ks * kTileBytes);
#pragma unroll 1
        for (int kk = 0; kk < ksteps; ++kk) mma_ss(tmem + TM_S, kd + 128 * kk, vd + 128 * kk, kIdescSU, 1u);
      };
      // O += phi(Q) S_{b-1} (A = phi(Q) in TMEM, B = the bf16 snapshot).
      auto issue_qs = [&](uint32_t qs) {
        const uint64_t sd = desc_at(kDescMN, sbase + OFF_SNAP);
#pragma unroll 1
        for (int kk = 0; kk < 8; ++kk) mma_ts(tmem + TM_O, tmem + TM_Q + 64 * qs + 8 * kk, sd + 128 * kk, kIdesc128MN, 1u);
      };

      // Per block, score jobs A = Q0 K0^T (masked), B = Q1 K0^T (dense), C = Q1 K1^T (masked)
      // run back to back through the one score region: each job is issued right after the
      // previous job's PV, so the conversion warps always have the next job in flight, and
      // the inter products and state updates fill the tensor pipe while they convert.  Tile
      // 0's accumulator is PV_A + Q0 S_{b-1}; tile 1's is PV_B + PV_C + Q1 S_{b-1}.  Each
      // operand is released after its last use: K0 after B and the state update over tile 0,
      // V0 after PV_B, K1 after C and the update over tile 1, V1 after PV_C.  su_done comes
      // after both inter products, so the snapshot area is free once the state warps see it.
      for (; it.valid && ok; blk_next<tpb>(p, it, wk)) {
        int vr0, vr1;
        const int n = blk_tiles<tpb, kRev>(it, vr0, vr1);
        const uint32_t s0 = ot & 1u, s1 = (ot + 1) & 1u;            // slots (and phi(Q) tiles)
        const uint32_t ph0 = (ot >> 1) & 1u, ph1 = ((ot + 1) >> 1) & 1u;
        const int pad0 = pad_rows(vr0), pad1 = n > 1 ? pad_rows(vr1) : 0;
        if (!mw(&B.xf_k[s0], ph0, ot) || !mw(&B.qt_ready[s0], ph0, ot)) break;
        issue_p(s0, s0, static_cast<uint32_t>(pad0));                                   // A
        if (!mw(&B.full_v[s0], ph0, ot)) break;
        if (ot >= 1 && !mw(&B.o_empty, (ot - 1) & 1u, ot)) break;
        if (!issue_pv(s0, pad0 / 16, false)) break;                                     // PV_A
        if (n > 1) {
          if (!mw(&B.qt_ready[s1], ph1, ot + 1)) break;
          issue_p(s1, s0, static_cast<uint32_t>(pad0));                                 // B
        }
        if (!mw(&B.snap_ready, nb & 1u, nb)) break;
        issue_qs(s0);
        mma_commit(&B.o_full);
        mma_commit(&B.qt_free[s0]);
        if (!mw(&B.s_ready, nb & 1u, nb)) break;
        issue_su(s0, pad0 / 16);
        mma_commit(&B.k_empty[s0]);
        if (n > 1) {
          if (!mw(&B.o_empty, ot & 1u, ot + 1)) break;   // the drain warps have read tile 0
          if (!issue_pv(s0, pad0 / 16, false)) break;                                   // PV_B
          mma_commit(&B.v_empty[s0]);
          if (!mw(&B.xf_k[s1], ph1, ot + 1)) break;
          issue_p(s1, s1, static_cast<uint32_t>(pad1));                                 // C
          if (!mw(&B.full_v[s1], ph1, ot + 1)) break;
          issue_su(s1, pad1 / 16);
          mma_commit(&B.k_empty[s1]);
          if (!issue_pv(s1, pad1 / 16, true)) break;                                    // PV_C
          mma_commit(&B.v_empty[s1]);
          issue_qs(s1);
          mma_commit(&B.o_full);
          mma_commit(&B.qt_free[s1]);
        } else {
          mma_commit(&B.v_empty[s0]);
        }
        mma_commit(&B.su_done);
        ot += n;
        ++nb;
      }
      // Drain: all MMAs complete before TMEM is released.
      mma_commit(&B.final_bar);
      tcu::drain(&B.final_bar, 0);
    }
  }
  // ------------------------------------------------------------------------------------
  // Warps 2, 3, 24-31: SiLU of this CTA's K tiles in place (tail rows of K zeroed, and of V once it
  // has landed).
  // ------------------------------------------------------------------------------------
  else if (warp == 2 || warp == 3 || warp >= kXfWarp1) {
    const int wt = warp < kXfWarp1 ? tid - 64 : tid - 32 * kXfWarp1 + 64;
    const bool silu = !p.phi_identity;
    uint32_t ot = 0;
    BlkIter it;
    blk_first<tpb>(p, it, wk);
    for (; it.valid; blk_next<tpb>(p, it, wk)) {
      int vr0, vr1;
      const int n = blk_tiles<tpb, kRev>(it, vr0, vr1);
      bool ok = true;
      for (int u = 0; u < n && ok; ++u) {
        const uint32_t t = ot + u, sl = t & 1u;
        const int vr = u == 0 ? vr0 : vr1;
        ok = tcu::wait_warp(&B.full_k[sl], (t >> 1) & 1u, abort_flag, err, SITE_TC_TRANSFORM, t);
        if (!ok) break;
        xf_tile(sbase + OFF_K + sl * kTileBytes, vr, silu, wt);
        if (vr < kTile) {
          ok = tcu::wait_warp(&B.full_v[sl], (t >> 1) & 1u, abort_flag, err, SITE_TC_TRANSFORM, t);
          if (!ok) break;
          zero_tail(sbase + OFF_V + sl * kTileBytes, vr, wt);
        }
        fence_proxy_async_smem();
        mbar_arrive(&B.xf_k[sl]);
      }
      if (!ok) break;
      ot += n;
    }
  }
  // ------------------------------------------------------------------------------------
  // Warps 8-11: SiLU of this CTA's Q tiles into TMEM (the A operand of the score and inter
  // MMAs); thread r converts row r of the tile (16 swizzled 16-byte chunks) and writes its
  // 64 columns of bf16 pairs.  The landing slot is free once read.
  // ------------------------------------------------------------------------------------
  else if (warp >= kQxfWarp0 && warp < kQxfWarp0 + 4) {
    const int r = tid - 32 * kQxfWarp0;
    const uint32_t tq = tmem + (static_cast<uint32_t>(r & ~31) << 16) + TM_Q;
    const bool silu = !p.phi_identity;
    uint32_t ot = 0;
    BlkIter it;
    blk_first<tpb>(p, it, wk);
    bool ok = true;
    for (; it.valid && ok; blk_next<tpb>(p, it, wk)) {
      int vr0, vr1;
      const int n = blk_tiles<tpb, kRev>(it, vr0, vr1);
      for (int u = 0; u < n; ++u) {
        const uint32_t t = ot + u, sl = t & 1u;   // landing slot and phi(Q) tile in TMEM
        if (!tcu::wait_warp(&B.full_q[sl], (t >> 1) & 1u, abort_flag, err, SITE_TC_TRANSFORM, t) ||
            (t >= 2 && !tcu::wait_warp(&B.qt_free[sl], ((t >> 1) - 1) & 1u, abort_flag, err, SITE_TC_TRANSFORM, t))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t src = sbase + OFF_Q + sl * kTileBytes;
#pragma unroll 1
        for (int g = 0; g < 4; ++g) {   // 32 columns of d_k: chunks 4g .. 4g + 3 of the row
          uint32_t x[16];
#pragma unroll
          for (int m4 = 0; m4 < 4; ++m4) {
            const int m = 4 * g + m4;   // 8-column chunk of the row (box m / 8)
            uint4 v = lds128(src + (m >> 3) * kBoxBytes + sw128_offset(r, m & 7));
            if (silu) v = tcu::silu8(v);
            x[4 * m4] = v.x; x[4 * m4 + 1] = v.y; x[4 * m4 + 2] = v.z; x[4 * m4 + 3] = v.w;
          }
          tmem_st16(tq + 64 * sl + 16 * g, x);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if ((r & 31) == 0) {
          mbar_arrive(&B.q_empty[sl]);
          mbar_arrive(&B.qt_ready[sl]);
        }
      }
      ot += n;
    }
  }
  // ------------------------------------------------------------------------------------
  // Warps 4-7: score conversion (fp32 -> masked bf16 in place in TMEM), job by job; thread
  // r owns row r of the score tile.
  // ------------------------------------------------------------------------------------
  else if (warp >= kConvWarp0 && warp < kConvWarp0 + 4) {
    const int r = tid - 32 * kConvWarp0;
    const uint32_t lane_t = tmem + (static_cast<uint32_t>(r & ~31) << 16);
    uint32_t uc = 0;   // score jobs converted
    bool ok = true;
    auto conv = [&](int ncols, bool diag) -> bool {
      const uint32_t tP = lane_t + TM_P;
      if (!tcu::wait_warp(&B.p_full, uc & 1u, abort_flag, err, SITE_TC_CONVERT, uc)) return false;
      tc_fence_after();
      for (int c = 0; c < ncols / 32; ++c) {
        uint32_t x[32];
        tmem_ld32(tP + 32 * c, x);
        tmem_ld_wait();
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int j = 32 * c + 16 * hh + 2 * e;
            float a = __uint_as_float(x[16 * hh + 2 * e]), b = __uint_as_float(x[16 * hh + 2 * e + 1]);
            if (diag) {   // keys up to the query row; from it on when time runs backwards
              a = (kRev ? j >= r : j <= r) ? a : 0.f;
              b = (kRev ? j + 1 >= r : j + 1 <= r) ? b : 0.f;
            }
            pk[e] = pack_bf16x2(a, b);
          }
          tmem_st8(tP + 16 * c + 8 * hh, pk);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&B.p_conv);
      ++uc;
      return true;
    };
    BlkIter it;
    blk_first<tpb>(p, it, wk);
    for (; it.valid && ok; blk_next<tpb>(p, it, wk)) {
      int vr0, vr1;
      const int n = blk_tiles<tpb, kRev>(it, vr0, vr1);
      // jobs A (tile 0, masked), then for two tiles B (dense, over tile 0's keys) and C (tile
      // 1, masked); going backwards in time tile 0 may be the sequence's partial tile
#pragma unroll 1
      for (int j = 0; j < 2 * n - 1 && ok; ++j) ok = conv(j == 1 ? pad_rows(vr0) : pad_rows(j == 0 ? vr0 : vr1), j != 1);
    }
  }
  // ------------------------------------------------------------------------------------
  // Warps 12-15 (one per TMEM lane quarter; thread r owns row r of every TMEM tile):
  //  * the state: S0 into TMEM and the bf16 snapshot at a sequence start; after each
  //    block's state update, S_b once: into the snapshot for the next block's inter
  //    products, or to state_out after the sequence's last block;
  //  * the output accumulators: each tile's rows read once and written out (y, or z for the
  //    final warps to rescale), and in the norm modes the rows' sums of squares published.
  // Per block: tile 0 (read, then published), tile 1 (read), the state, tile 1's sums -- the
  // order in which the MMA warp makes them ready, reads that free the accumulator first.
  // ------------------------------------------------------------------------------------
  else if (warp >= kStateWarp0 && warp < kStateWarp0 + 4) {
    const int r = tid - 32 * kStateWarp0;          // TMEM lane: row of a tile, or d_k row of S
    const uint32_t lane_off = static_cast<uint32_t>(r & ~31) << 16;
    const uint32_t tS = tmem + lane_off + TM_S;
    const uint32_t snap = sbase + OFF_SNAP;
    const bool skip_publish = (err->inject == INJECT_SKIP_PUBLISH) && blockIdx.x == 0;
    uint32_t nb = 0, ot = 0;
    bool ok = true;
    // Drain own tile t (tile i of the block's sequence): read row r of the accumulator once,
    // free it, and write the row to the output -- y in raw mode, z = bf16(y w) in the norm
    // modes, where the final warps rescale it in place -- then publish the row's sum of
    // squares (fp64 add into the token's total, fence, one arrival per warp).
    const int64_t HD = static_cast<int64_t>(p.H) * kD;
    // drain() reads tile t's row r and frees the accumulator; publish() then adds the row's
    // sum of squares (kept in ss_row) and makes the warp's arrival.
    float ss_row = 0.f;
    auto drain = [&](uint32_t t, const BlkIter& bi, int u, int vr) -> bool {
      if (!tcu::wait_warp(&B.o_full, t & 1u, abort_flag, err, SITE_TC_EPILOGUE, t)) return false;
      tc_fence_after();
      const int i = bi.jb * tpb + u;
      const int64_t row = bi.row0 + static_cast<int64_t>(phys_tile<kRev>(i, bi.nt)) * kTile + r;
      const bool valid = r < vr;
      uint16_t* dst = p.out + row * HD + h * kD;
      float ss = 0.f;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t x[16];
        tmem_ld16(tmem + lane_off + TM_O + 16 * c, x);
        tmem_ld_wait();
        uint32_t z[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float a = __uint_as_float(x[2 * e]), b = __uint_as_float(x[2 * e + 1]);
          ss = fmaf(a, a, ss);
          ss = fmaf(b, b, ss);
          if (norm) {
            a *= B.w[16 * c + 2 * e];
            b *= B.w[16 * c + 2 * e + 1];
          }
          z[e] = pack_bf16x2(a, b);
        }
        if (valid) tcu::st_na_v8(dst + 16 * c, z);
      }
      tc_fence_before();
      __syncwarp();
      if ((r & 31) == 0) mbar_arrive(&B.o_empty);   // done reading the accumulator
      ss_row = ss;
      return true;
    };
    auto publish = [&](const BlkIter& bi, int u, int vr) {
      if (!norm) return;
      const int i = bi.jb * tpb + u;
      const int64_t row = bi.row0 + static_cast<int64_t>(phys_tile<kRev>(i, bi.nt)) * kTile + r;
      if (r < vr) tcu::red_add_f64(p.ss + row * kSsStride, static_cast<double>(ss_row));
      tcu::fence_acq_rel_gpu();
      __syncwarp();
      if ((r & 31) == 0 && !skip_publish)
        tcu::red_add_relaxed_u32(p.cnt + (static_cast<int64_t>(bi.s) * p.max_tiles + i) * kCntStride, 1u);
    };
    // Columns 16c .. 16c + 15 of row r of S into the snapshot (two 16-byte bf16 chunks).
    auto snap16 = [&](int c, const uint32_t (&x)[16]) {
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int m = 2 * c + h2;   // 8-column chunk of the row
        const uint32_t* a = x + 8 * h2;
        sts128(snap + (m >> 3) * kBoxBytes + sw128_offset(r, m & 7),
               make_uint4(pack_bf16x2(__uint_as_float(a[0]), __uint_as_float(a[1])),
                          pack_bf16x2(__uint_as_float(a[2]), __uint_as_float(a[3])),
                          pack_bf16x2(__uint_as_float(a[4]), __uint_as_float(a[5])),
                          pack_bf16x2(__uint_as_float(a[6]), __uint_as_float(a[7]))));
      }
    };
    // State slots: state_in by the sequence's slot; state_out by its slot, or for chunks by
    // the sequence it ends (a chunk that is not its sequence's last writes nothing).
    auto in_row = [&](int s) -> int64_t {
      const int64_t slot = p.state_index ? __ldg(p.state_index + s) : s;
      return ((slot * p.H + h) * kD + r) * kD;
    };
    auto out_row = [&](int s) -> int64_t {
      if (!p.state_out) return -1;
      int64_t slot = s;
      if (p.state_index) slot = __ldg(p.state_index + s);
      else if (p.chunk_div > 1) {   // the chunk that ends the walk holds the sequence's final state
        if (s % p.chunk_div != (kRev ? 0 : p.chunk_div - 1)) return -1;
        slot = s / p.chunk_div;
      }
      return ((slot * p.H + h) * kD + r) * kD;
    };
    // Empty sequences of this worker: S0 is their final state.
    {
      int k0, k1;
      worker_range(p, wk, k0, k1);
      for (int k = k0; k < k1; ++k) {
        const int s = worker_seq(p, wk, k);
        int64_t r0;
        int L;
        if (seq_range(p, s, r0, L) || L > 0) continue;
        const int64_t o = out_row(s);
        if (o < 0) continue;
        const int64_t ir = in_row(s);
        for (int c = 0; c < kD; c += 4) {
          const float4 x = p.state_in ? *reinterpret_cast<const float4*>(p.state_in + ir + c) : make_float4(0, 0, 0, 0);
          *reinterpret_cast<float4*>(p.state_out + o + c) = x;
        }
      }
    }
    BlkIter it;
    blk_first<tpb>(p, it, wk);
    for (; it.valid && ok; blk_next<tpb>(p, it, wk)) {
      int vr0, vr1;
      const int n = blk_tiles<tpb, kRev>(it, vr0, vr1);
      const bool first = it.jb == 0, last = it.jb == it.nblk - 1;
      if (first) {   // S0 into TMEM and the snapshot
        const int64_t ir = in_row(it.s);
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t x[16];
#pragma unroll
          for (int j = 0; j < 16; j += 4) {
            const float4 v = p.state_in ? *reinterpret_cast<const float4*>(p.state_in + ir + 16 * c + j)
                                        : make_float4(0, 0, 0, 0);
            x[j] = __float_as_uint(v.x); x[j + 1] = __float_as_uint(v.y);
            x[j + 2] = __float_as_uint(v.z); x[j + 3] = __float_as_uint(v.w);
          }
          tmem_st16(tS + 16 * c, x);
          snap16(c, x);
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&B.snap_ready);
        mbar_arrive(&B.s_ready);
      }
      if (!drain(ot, it, 0, vr0)) break;
      publish(it, 0, vr0);
      if (n > 1 && !drain(ot + 1, it, 1, vr1)) break;
      // S_b, once the block's state update is done
      if (!tcu::wait_warp(&B.su_done, nb & 1u, abort_flag, err, SITE_TC_EPILOGUE, nb)) break;
      tc_fence_after();
      const int64_t o = last ? out_row(it.s) : -1;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t x[16];
        tmem_ld16(tS + 16 * c, x);
        tmem_ld_wait();
        if (!last) {
          snap16(c, x);
        } else if (o >= 0) {
#pragma unroll
          for (int j = 0; j < 16; j += 4)
            *reinterpret_cast<float4*>(p.state_out + o + 16 * c + j) =
                make_float4(__uint_as_float(x[j]), __uint_as_float(x[j + 1]), __uint_as_float(x[j + 2]),
                            __uint_as_float(x[j + 3]));
        }
      }
      tc_fence_before();
      if (!last) {
        fence_proxy_async_smem();
        mbar_arrive(&B.snap_ready);
        mbar_arrive(&B.s_ready);
      }
      ++nb;
      if (n > 1) publish(it, 1, vr1);
      ot += n;
    }
  }
  // ------------------------------------------------------------------------------------
  // Warps 16-23 (norm modes): the normalised output.  Once every head has published a
  // tile's sums, its rows (z = bf16(y w), written by the drain warps) are rescaled in place:
  // o = z rsqrt(mean(y^2) + eps) [sigmoid(g)].  No TMEM access: warp e takes rows
  // 16e .. 16e + 15 of the tile, each half-warp one row's 256 bytes of this head per step,
  // so every access is a full 512-byte line pair.
  // ------------------------------------------------------------------------------------
  else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kEpiWarps && norm) {
    const int e = warp - kEpiWarp0;
    const int half = lane >> 4;                       // which row of the pair
    const int cl = (lane & 15) * 8;                   // this lane's 8 columns of the head
    const int64_t HD = static_cast<int64_t>(p.H) * kD;
    const float inv_hd = 1.0f / static_cast<float>(HD);
    uint32_t ot = 0;
    bool ok = true;
    BlkIter it;
    blk_first<tpb>(p, it, wk);
    for (; it.valid && ok; blk_next<tpb>(p, it, wk)) {
      int vr0, vr1;
      const int n = blk_tiles<tpb, kRev>(it, vr0, vr1);
      for (int u = 0; u < n && ok; ++u, ++ot) {
        const int i = it.jb * tpb + u;                 // tile of the sequence
        const int vr = u == 0 ? vr0 : vr1;
        unsigned int* cnt = p.cnt + (static_cast<int64_t>(it.s) * p.max_tiles + i) * kCntStride;
        int go = 1;
        if (lane == 0 && ld_acquire_gpu(cnt) < W)
          go = tcu::poll_count(cnt, W, abort_flag, err, static_cast<uint32_t>(it.s * p.max_tiles + i)) ? 1 : 0;
        if (!__shfl_sync(0xFFFFFFFFu, go, 0)) {
          ok = false;
          break;
        }
        (void)ld_acquire_gpu(cnt);
        const int64_t base = it.row0 + static_cast<int64_t>(phys_tile<kRev>(i, it.nt)) * kTile;
        // Lane l holds the norm factor of row 16e + (l & 15).
        const int myrt = 16 * e + (lane & 15);
        const double myss = myrt < vr ? tcu::ld_cg_f64(p.ss + (base + myrt) * kSsStride) : 0.0;
        const float myrn = 1.0f / sqrtf(static_cast<float>(myss) * inv_hd + p.eps);
        const uint16_t* zrow = p.out + (base + 16 * e + half) * HD + h * kD + cl;   // row pair 0
        const uint16_t* grow = gate ? p.g + (base + 16 * e + half) * HD + h * kD + cl : nullptr;
#pragma unroll 1
        for (int k0 = 0; k0 < 8; k0 += 2) {           // 2 row pairs at a time
          uint4 zv[2], gv[2];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int rt = 16 * e + 2 * (k0 + k) + half;   // row of the tile
            const bool valid = rt < vr;
            const int64_t off = static_cast<int64_t>(2 * (k0 + k)) * HD;
            zv[k] = valid ? tcu::ld_cg_u4(zrow + off) : make_uint4(0, 0, 0, 0);
            gv[k] = (gate && valid) ? tcu::ld_nc_u4(grow + off) : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int rt = 16 * e + 2 * (k0 + k) + half;
            const float rn = __shfl_sync(0xFFFFFFFFu, myrn, 2 * (k0 + k) + half);
            if (rt >= vr) continue;
            const uint32_t zw[4] = {zv[k].x, zv[k].y, zv[k].z, zv[k].w};
            const uint32_t gw[4] = {gv[k].x, gv[k].y, gv[k].z, gv[k].w};
            uint32_t o[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float a = __uint_as_float(zw[q] << 16) * rn, b = __uint_as_float(zw[q] & 0xFFFF0000u) * rn;
              if (gate) {
                a *= sigmoid_fast(__uint_as_float(gw[q] << 16));
                b *= sigmoid_fast(__uint_as_float(gw[q] & 0xFFFF0000u));
              }
              o[q] = pack_bf16x2(a, b);
            }
            tcu::st_global_na(const_cast<uint16_t*>(zrow) + static_cast<int64_t>(2 * (k0 + k)) * HD,
                              make_uint4(o[0], o[1], o[2], o[3]));
          }
        }
      }
    }
  }

  // Teardown: every role is done (or aborted with its async work drained).  The cluster
  // barrier keeps this CTA's shared memory alive until the partner has stopped arriving on
  // its barriers.
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc<kTmemCols>(tmem);
}

// ======================================================================================
// Host side
// ======================================================================================
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [rows, cols] bf16 row-major, box 64 columns x 128 rows, 128-byte swizzle, zero fill.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kTile)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

inline size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

using PairKernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, PairParams);
PairKernel pair_kernel(int mode, int C, bool rev) {
  static const PairKernel k[4][2] = {
      {lightning_prefill_pair_kernel<LA_OUT_RAW, 128, false>, lightning_prefill_pair_kernel<LA_OUT_RAW, 256, false>},
      {lightning_prefill_pair_kernel<LA_OUT_RMSNORM, 128, false>,
       lightning_prefill_pair_kernel<LA_OUT_RMSNORM, 256, false>},
      {lightning_prefill_pair_kernel<LA_OUT_RMSNORM_GATE, 128, false>,
       lightning_prefill_pair_kernel<LA_OUT_RMSNORM_GATE, 256, false>},
      {lightning_prefill_pair_kernel<LA_OUT_RAW, 128, true>, lightning_prefill_pair_kernel<LA_OUT_RAW, 256, true>}};
  const int m = rev ? 3 : (mode == LA_OUT_RAW ? 0 : (mode == LA_OUT_RMSNORM ? 1 : 2));
  return k[m][C == 256 ? 1 : 0];
}

}  // namespace

// CTA pairs of this kernel that fit on the current device at once; cached per device.
int pair_max_active_clusters() {
  static int cache[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    PairKernel kern = pair_kernel(LA_OUT_RMSNORM_GATE, 256, false);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemBytes)) !=
        cudaSuccess)
      return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = -1;
    cache[dev] = n;
  }
  return cache[dev];
}

// Sequence groups of a call: with few heads, the CTA pairs of several groups split the
// sequences, as many groups as fit at once (the norm exchange needs all pairs resident).
int pair_groups(int nseq, int H) {
  const int maxc = pair_max_active_clusters();
  return maxc > H ? std::max(1, std::min(nseq, maxc / H)) : 1;
}

namespace {

constexpr int kPlanMaxSeqs = 2048;   // packed batches up to this size get a longest-first plan
constexpr int kPlanThreads = 1024;

// The worker plan of a packed batch: sequences sorted by length, longest first (bitonic
// sort in shared memory), then dealt to the 2G workers: each to the least-loaded worker
// (LPT) for up to 256 sequences, in snake order beyond.  sched lists the sequences worker by
// worker (longest first within a worker); wstart[w] is worker w's first entry.  Every head
// uses the same plan, so the same worker of every head walks the same tiles.
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const int* __restrict__ cu, int nseq, int nw,
                                                            int skip_single, int* __restrict__ sched,
                                                            int* __restrict__ wstart) {
  __shared__ unsigned long long key[kPlanMaxSeqs];
  __shared__ int owner[kPlanMaxSeqs];
  __shared__ long long load[256];
  __shared__ int count[257];
  int n2 = 1;
  while (n2 < nseq) n2 <<= 1;
  for (int i = threadIdx.x; i < n2; i += blockDim.x) {
    unsigned long long k = 0;
    if (i < nseq) {
      int L = __ldg(cu + i + 1) - __ldg(cu + i);
      if (L < 0 || (skip_single && L == 1)) L = 0;
      // length in the high word; ties keep the lower index first
      k = (static_cast<unsigned long long>(L) << 32) | (0xFFFFFFFFu - static_cast<unsigned>(i));
    }
    key[i] = k;
  }
  for (int w = threadIdx.x; w < 257; w += blockDim.x) count[w] = 0;
  for (int w = threadIdx.x; w < 256; w += blockDim.x) load[w] = 0;
  __syncthreads();
  for (int size = 2; size <= n2; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < n2; i += blockDim.x) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0;   // descending overall
          const unsigned long long a = key[i], b = key[j];
          if (desc ? (a < b) : (a > b)) {
            key[i] = b;
            key[j] = a;
          }
        }
      }
      __syncthreads();
    }
  // Assignment of sorted position i to a worker.
  if (nseq <= 256) {
    if (threadIdx.x < 32) {
      for (int i = 0; i < nseq; ++i) {
        long long best = LLONG_MAX;
        int bw = 0;
        for (int w = threadIdx.x; w < nw; w += 32)
          if (load[w] < best) { best = load[w]; bw = w; }
        for (int off = 16; off > 0; off >>= 1) {
          const long long ob = __shfl_down_sync(0xFFFFFFFFu, best, off);
          const int ow = __shfl_down_sync(0xFFFFFFFFu, bw, off);
          if (ob < best || (ob == best && ow < bw)) { best = ob; bw = ow; }
        }
        bw = __shfl_sync(0xFFFFFFFFu, bw, 0);
        if (threadIdx.x == 0) {
          owner[i] = bw;
          load[bw] += static_cast<long long>(key[i] >> 32) + 1;
        }
        __syncwarp();
      }
    }
  } else {
    for (int i = threadIdx.x; i < nseq; i += blockDim.x) {
      const int round = i / nw, pos = i % nw;
      owner[i] = (round & 1) ? nw - 1 - pos : pos;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 0; i < nseq; ++i) count[owner[i] + 1]++;
    for (int w = 0; w < nw; ++w) count[w + 1] += count[w];
    for (int w = 0; w <= nw; ++w) wstart[w] = count[w];
    for (int i = 0; i < nseq; ++i) sched[count[owner[i]]++] = static_cast<int>(0xFFFFFFFFu - static_cast<unsigned>(key[i] & 0xFFFFFFFFull));
  }
}

}  // namespace

// Workspace after the error record: [arrival counters] [fp64 sums] [plan: sched, wstart].
size_t pair_workspace_bytes(int nseq, int max_len, int64_t tokens, int H) {
  const size_t max_tiles = (static_cast<size_t>(max_len) + kTile - 1) / kTile;
  const size_t nw = 2 * static_cast<size_t>(pair_groups(nseq, H));
  return up256(sizeof(unsigned int) * kCntStride * static_cast<size_t>(nseq) * (max_tiles ? max_tiles : 1)) +
         up256(sizeof(double) * kSsStride * static_cast<size_t>(tokens > 0 ? tokens : 1)) +
         up256(sizeof(int) * static_cast<size_t>(nseq)) + up256(sizeof(int) * (nw + 1));
}

cudaError_t launch_pair_prefill(const TcArgs& a, cudaStream_t stream) {
  if (a.D != kD || (a.C != 128 && a.C != 256) || (a.reverse && a.mode != LA_OUT_RAW)) return cudaErrorInvalidValue;
  const int max_tiles = (a.max_len + kTile - 1) / kTile;
  const size_t cnt_bytes =
      up256(sizeof(unsigned int) * kCntStride * static_cast<size_t>(a.nseq) * (max_tiles ? max_tiles : 1));
  const size_t ss_bytes = up256(sizeof(double) * kSsStride * static_cast<size_t>(a.tokens > 0 ? a.tokens : 1));
  const size_t sched_bytes = up256(sizeof(int) * static_cast<size_t>(a.nseq));
  PairParams p{};
  p.state_in = a.state_in;
  p.state_out = a.state_out;
  p.cu = a.cu;
  p.nseq = a.nseq;
  p.T = a.T;
  p.H = a.H;
  p.phi_identity = a.phi_identity;
  p.max_tiles = max_tiles;
  p.chunk_div = a.chunk_div > 1 ? a.chunk_div : 1;
  p.tokens = a.tokens;
  p.eps = a.eps;
  p.w = a.w;
  p.g = static_cast<const uint16_t*>(a.g);
  p.state_index = a.state_index;
  p.skip_single = a.skip_single;
  p.err = a.err;
  p.cnt = reinterpret_cast<unsigned int*>(a.ws);
  p.ss = reinterpret_cast<double*>(a.ws + cnt_bytes);
  p.out = static_cast<uint16_t*>(a.out);
  p.ngroups = pair_groups(a.nseq, a.H);
  const int nw = 2 * p.ngroups;

  const int64_t cols = static_cast<int64_t>(a.H) * kD;
  CUtensorMap mq, mk, mv, mg;
  if (!make_map(&mq, a.q, a.tokens, cols) || !make_map(&mk, a.k, a.tokens, cols) ||
      !make_map(&mv, a.v, a.tokens, cols))
    return cudaErrorInvalidValue;
  if (a.mode == LA_OUT_RMSNORM_GATE) {
    if (!make_map(&mg, a.g, a.tokens, cols)) return cudaErrorInvalidValue;
  } else {
    mg = mq;   // never read
  }
  // Arrival counters and the fp64 sums start at zero on every call.
  cudaError_t e = cudaMemsetAsync(a.ws, 0, cnt_bytes + (a.mode != LA_OUT_RAW ? ss_bytes : 0), stream);
  if (e != cudaSuccess) return e;
  // Packed batches with more sequences than workers: the longest-first worker plan (with
  // at most one sequence per worker the round-robin order is already that plan).
  if (a.cu && a.nseq > nw && a.nseq <= kPlanMaxSeqs && nw <= 256) {
    int* sched = reinterpret_cast<int*>(a.ws + cnt_bytes + ss_bytes);
    int* wstart = reinterpret_cast<int*>(a.ws + cnt_bytes + ss_bytes + sched_bytes);
    plan_kernel<<<1, kPlanThreads, 0, stream>>>(a.cu, a.nseq, nw, a.skip_single, sched, wstart);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    p.sched = sched;
    p.wstart = wstart;
  }
  const PairKernel kernel = pair_kernel(a.mode, a.C, a.reverse != 0);
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * a.H * p.ngroups);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kernel, mq, mk, mv, mg, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace la
