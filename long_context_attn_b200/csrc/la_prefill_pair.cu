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
//  * Roles (24 warps): warp 0 streams Q tiles (lane 0) and K/V tiles (lane 1) with TMA into
//    two-slot rings; warp 1 issues every MMA; warps 2-7 apply SiLU (packed bf16x2
//    arithmetic) to Q and K in place; warps 8-11 turn score tiles into masked bf16 in TMEM;
//    warps 12-15 own the state (S0 in, the snapshot, the final state out); warps 16-23 read
//    the output accumulators (each warp 64 of the 128 columns of its TMEM lane quarter),
//    publish the rows' sums of squares and, once all heads of the tile have published,
//    read the accumulator again and store o = y w rsqrt(mean(y^2) + eps) sigmoid(g).
//  * TMEM (512 columns): S (128), two output accumulators (2 x 128), one score region (128).
//  * Cross-head RMSNorm: every epilogue thread adds its row's partial sum of squares into an
//    fp64 per-token total (red.add; exact and order-independent while a token's partials
//    span less than 2^22), and each warp bumps the tile's arrival counter after a fence.
//    The same worker of every head processes the same tiles in the same order, and all CTAs
//    are resident at once (checked on the host).
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
constexpr int kThreads = 768;     // 24 warps
constexpr int kConvWarp0 = 4;     // warps 4..7: score conversion, the state, the rows' sums of squares
constexpr int kXfThreads = 320;   // transform: warps 2, 3 and 8..15
constexpr int kXfIlp = 8;         // 16-byte chunks in flight per transform thread
constexpr int kEpiWarp0 = 16;     // warps 16..23: the output stores
constexpr int kEpiWarps = 8;
constexpr int kPubWarps = 4;      // arrivals per CTA that publish a tile's sums

constexpr uint32_t kBoxBytes = kTile * 64 * 2;    // one 128-row x 64-column bf16 box (16 KiB)
constexpr uint32_t kTileBytes = 2 * kBoxBytes;    // a 128 x 128 tile: two boxes (32 KiB)
constexpr uint32_t OFF_Q = 0;                     // 2 slots
constexpr uint32_t OFF_K = OFF_Q + 2 * kTileBytes;
constexpr uint32_t OFF_V = OFF_K + 2 * kTileBytes;
constexpr uint32_t OFF_SNAP = OFF_V + 2 * kTileBytes;
constexpr uint32_t OFF_BARS = OFF_SNAP + kTileBytes;

constexpr uint32_t TM_S = 0;      // S, 128 columns (lanes = d_k, columns = d_v)
constexpr uint32_t TM_O = 128;    // two output accumulators, 128 columns each
constexpr uint32_t TM_P = 384;    // score region, 128 columns
constexpr uint32_t kTmemCols = 512;

struct Bars {
  uint64_t full_q[2], xf_q[2], q_empty[2];
  uint64_t full_kv[2], xf_kv[2], kv_empty[2];
  uint64_t p_full, p_conv, pv_done;
  uint64_t o_full[2], o_empty[2];
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
// Tiles of the current block and the valid rows of each.
template <int tpb>
__device__ __forceinline__ int blk_tiles(const BlkIter& it, int& vr0, int& vr1) {
  const int t0 = it.jb * tpb;
  const int n = min(tpb, it.nt - t0);
  vr0 = min(kTile, it.L - t0 * kTile);
  vr1 = n > 1 ? min(kTile, it.L - (t0 + 1) * kTile) : 0;
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
template <int kMode, int kC>
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
      mbar_init(&B.full_q[i], 1);
      mbar_init(&B.xf_q[i], kXfThreads);
      mbar_init(&B.q_empty[i], 1);
      mbar_init(&B.full_kv[i], 1);
      mbar_init(&B.xf_kv[i], kXfThreads);
      mbar_init(&B.kv_empty[i], 1);
      mbar_init(&B.o_full[i], 1);
      mbar_init(&B.o_empty[i], kEpiWarps);
    }
    mbar_init(&B.p_full, 1);
    mbar_init(&B.p_conv, 128);
    mbar_init(&B.pv_done, 1);
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
  // Warp 0: TMA producers.  Lane 0: Q tiles of this CTA's blocks into Q slot (own tile % 2);
  // lane 1: K and V tiles into K/V slot (own tile % 2), and the gate tile prefetched into
  // L2 for the epilogue.  Own tiles are numbered in walk order; both rings use that number.
  // ------------------------------------------------------------------------------------
  if (warp == 0) {
    if (lane < 2) {
      const bool is_q = lane == 0;
      if (is_q) {
        prefetch_tmap(&tm_q);
      } else {
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        if (gate) prefetch_tmap(&tm_g);
      }
      const uint64_t pol = policy_evict_first();
      uint32_t ot = 0;
      bool ok = true;
      BlkIter it;
      blk_first<tpb>(p, it, wk);
      for (; it.valid && ok; blk_next<tpb>(p, it, wk)) {
        int vr0, vr1;
        const int n = blk_tiles<tpb>(it, vr0, vr1);
        for (int u = 0; u < n; ++u, ++ot) {
          const uint32_t sl = ot & 1u;
          uint64_t* empty = is_q ? &B.q_empty[sl] : &B.kv_empty[sl];
          if (ot >= 2 && !tcu::wait(empty, ((ot >> 1) - 1) & 1u, abort_flag, err, SITE_TC_PRODUCER, ot)) {
            ok = false;
            break;
          }
          const int32_t row = static_cast<int32_t>(it.row0 + static_cast<int64_t>(it.jb * tpb + u) * kTile);
          const int32_t col = h * kD;
          // The same tile of the next block, into L2: the demand on DRAM runs a block ahead
          // of the two-slot rings.
          const bool ahead = (it.jb * tpb + u + tpb) < it.nt;
          if (is_q) {
            if (ahead) {
              tma_prefetch_l2_2d(&tm_q, col, row + kC);
              tma_prefetch_l2_2d(&tm_q, col + 64, row + kC);
            }
            uint8_t* dst = smem + OFF_Q + sl * kTileBytes;
            mbar_arrive_expect_tx(&B.full_q[sl], kTileBytes);
            tma_load_2d(dst, &tm_q, col, row, &B.full_q[sl], pol);
            tma_load_2d(dst + kBoxBytes, &tm_q, col + 64, row, &B.full_q[sl], pol);
          } else {
            if (ahead) {
              tma_prefetch_l2_2d(&tm_k, col, row + kC);
              tma_prefetch_l2_2d(&tm_k, col + 64, row + kC);
              tma_prefetch_l2_2d(&tm_v, col, row + kC);
              tma_prefetch_l2_2d(&tm_v, col + 64, row + kC);
            }
            uint8_t* dk = smem + OFF_K + sl * kTileBytes;
            uint8_t* dv = smem + OFF_V + sl * kTileBytes;
            mbar_arrive_expect_tx(&B.full_kv[sl], 2 * kTileBytes);
            tma_load_2d(dk, &tm_k, col, row, &B.full_kv[sl], pol);
            tma_load_2d(dk + kBoxBytes, &tm_k, col + 64, row, &B.full_kv[sl], pol);
            tma_load_2d(dv, &tm_v, col, row, &B.full_kv[sl], pol);
            tma_load_2d(dv + kBoxBytes, &tm_v, col + 64, row, &B.full_kv[sl], pol);
            if (gate) {
              tma_prefetch_l2_2d(&tm_g, col, row);
              tma_prefetch_l2_2d(&tm_g, col + 64, row);
            }
          }
        }
      }
      // Drain: every issued load must land before the CTA may exit (the last load into
      // each slot is own tile ot - 1 or ot - 2).
      for (uint32_t sl = 0; sl < 2; ++sl) {
        if (ot <= sl) continue;
        const uint32_t t = ((ot - 1) & 1u) == sl ? ot - 1 : ot - 2;
        tcu::drain(is_q ? &B.full_q[sl] : &B.full_kv[sl], (t >> 1) & 1u);
      }
    }
  }
  // ------------------------------------------------------------------------------------
  // Warp 1: MMA issuer (one thread).
  // ------------------------------------------------------------------------------------
  else if (warp == 1) {
    if (lane == 0) {
      uint32_t ot = 0, jb = 0, nb = 0;
      bool ok = true;
      BlkIter it;
      blk_first<tpb>(p, it, wk);
      auto mw = [&](uint64_t* bar, uint32_t par, uint32_t idx) -> bool {
        if (!tcu::wait(bar, par, abort_flag, err, SITE_TC_MMA, idx)) return false;
        tc_fence_after();
        return true;
      };
      // Score job into the region (after the previous job's PV has completed).
      auto issue_p = [&](uint32_t qs, uint32_t ks, uint32_t n) -> bool {
        if (jb > 0 && !mw(&B.pv_done, (jb - 1) & 1u, jb)) return false;
        const uint64_t qd = desc_at(kDescK, sbase + OFF_Q + qs * kTileBytes);
        const uint64_t kd = desc_at(kDescK, sbase + OFF_K + ks * kTileBytes);
        const uint32_t idesc = make_idesc_bf16(128, n, 0, 0);
#pragma unroll 1
        for (int kk = 0; kk < 8; ++kk) mma_ss(tmem + TM_P, qd + kstep_k(kk), kd + kstep_k(kk), idesc, kk > 0);
        mma_commit(&B.p_full);
        return true;
      };
      // PV of the current job into accumulator od over ksteps key steps.
      auto issue_pv = [&](uint32_t od, uint32_t vs, int ksteps, bool acc) -> bool {
        if (!mw(&B.p_conv, jb & 1u, jb)) return false;
        const uint64_t vd = desc_at(kDescMN, sbase + OFF_V + vs * kTileBytes);
#pragma unroll 1
        for (int kk = 0; kk < ksteps; ++kk)
          mma_ts(od, tmem + TM_P + 8 * kk, vd + 128 * kk, kIdesc128MN, (acc || kk > 0) ? 1u : 0u);
        mma_commit(&B.pv_done);
        ++jb;
        return true;
      };
      // S += phi(K)^T V over the keys of one tile (S was set by the state warps).
      auto issue_su = [&](uint32_t ks, int ksteps) {
        const uint64_t kd = desc_at(kDescMN, sbase + OFF_K + ks * kTileBytes);
        const uint64_t vd = desc_at(kDescMN, sbase + OFF_V + ks * kTileBytes);
#pragma unroll 1
        for (int kk = 0; kk < ksteps; ++kk)
          mma_ss(tmem + TM_S, kd + 128 * kk, vd + 128 * kk, kIdescSU, 1u);
      };
      auto issue_qs = [&](uint32_t od, uint32_t qs) {
        const uint64_t qd = desc_at(kDescK, sbase + OFF_Q + qs * kTileBytes);
        const uint64_t sd = desc_at(kDescMN, sbase + OFF_SNAP);
#pragma unroll 1
        for (int kk = 0; kk < 8; ++kk) mma_ss(od, qd + kstep_k(kk), sd + 128 * kk, kIdesc128MN, 1u);
      };

      // Per block: the score jobs (A = Q0 K0^T masked, B = Q1 K0^T dense, C = Q1 K1^T
      // masked) through the single score region, each followed by its PV; the inter
      // products with the snapshot of S_{b-1}; the state update over both tiles' keys after
      // the inter products (so that su_done also covers them and the snapshot area is free
      // once the state warps see it).
      for (; it.valid && ok; blk_next<tpb>(p, it, wk)) {
        int vr0, vr1;
        const int n = blk_tiles<tpb>(it, vr0, vr1);
        const uint32_t s0 = ot & 1u, s1 = (ot + 1) & 1u;            // slots (and accumulators)
        const uint32_t ph0 = (ot >> 1) & 1u, ph1 = ((ot + 1) >> 1) & 1u;
        const int pad0 = pad_rows(vr0), pad1 = n > 1 ? pad_rows(vr1) : 0;
        const uint32_t od0 = tmem + TM_O + 128 * s0, od1 = tmem + TM_O + 128 * s1;
        // job A: Q0 K0^T (masked) -> PV into accumulator s0, then Q0 S_{b-1}
        if (!mw(&B.xf_kv[s0], ph0, ot) || !mw(&B.xf_q[s0], ph0, ot)) break;
        if (!issue_p(s0, s0, static_cast<uint32_t>(pad0))) break;
        if (ot >= 2 && !mw(&B.o_empty[s0], ((ot >> 1) - 1) & 1u, ot)) break;
        if (!issue_pv(od0, s0, pad0 / 16, false)) break;
        if (!mw(&B.snap_ready, nb & 1u, nb)) break;
        issue_qs(od0, s0);
        mma_commit(&B.o_full[s0]);
        mma_commit(&B.q_empty[s0]);
        if (n > 1) {
          // job B: Q1 K0^T (dense) -> PV into accumulator s1, then Q1 S_{b-1}
          if (!mw(&B.xf_q[s1], ph1, ot + 1)) break;
          if (!issue_p(s1, s0, 128u)) break;
          if (ot + 1 >= 2 && !mw(&B.o_empty[s1], (((ot + 1) >> 1) - 1) & 1u, ot + 1)) break;
          if (!issue_pv(od1, s0, 8, false)) break;
          issue_qs(od1, s1);
          // state update over tile 0's and tile 1's keys
          if (!mw(&B.s_ready, nb & 1u, nb)) break;
          issue_su(s0, pad0 / 16);
          mma_commit(&B.kv_empty[s0]);   // tile 0's keys and values: A, B, S all issued
          if (!mw(&B.xf_kv[s1], ph1, ot + 1)) break;
          issue_su(s1, pad1 / 16);
          mma_commit(&B.su_done);
          // job C: Q1 K1^T (masked) -> PV into accumulator s1
          if (!issue_p(s1, s1, static_cast<uint32_t>(pad1))) break;
          if (!issue_pv(od1, s1, pad1 / 16, true)) break;
          mma_commit(&B.o_full[s1]);
          mma_commit(&B.q_empty[s1]);
          mma_commit(&B.kv_empty[s1]);
        } else {
          if (!mw(&B.s_ready, nb & 1u, nb)) break;
          issue_su(s0, pad0 / 16);
          mma_commit(&B.su_done);
          mma_commit(&B.kv_empty[s0]);
        }
        ot += n;
        ++nb;
      }
      (void)ok;
      // Drain: all MMAs complete before TMEM is released.
      mma_commit(&B.final_bar);
      tcu::drain(&B.final_bar, 0);
    }
  }
  // ------------------------------------------------------------------------------------
  // Warps 2, 3, 8-15: SiLU of this CTA's K and Q tiles in place, in the order the MMAs need them
  // (K0, Q0, Q1, K1 of each block); tail rows of K and V zeroed.
  // ------------------------------------------------------------------------------------
  else if (warp == 2 || warp == 3 || (warp >= 8 && warp < 16)) {
    const int wt = warp < 4 ? tid - 64 : tid - 192;   // 0..63, then 64..319
    const bool silu = !p.phi_identity;
    uint32_t ot = 0;
    BlkIter it;
    blk_first<tpb>(p, it, wk);
    auto do_k = [&](uint32_t t, int vr) -> bool {
      const uint32_t sl = t & 1u;
      if (!tcu::wait_warp(&B.full_kv[sl], (t >> 1) & 1u, abort_flag, err, SITE_TC_TRANSFORM, t)) return false;
      xf_tile(sbase + OFF_K + sl * kTileBytes, vr, silu, wt);
      if (vr < kTile) zero_tail(sbase + OFF_V + sl * kTileBytes, vr, wt);
      fence_proxy_async_smem();
      mbar_arrive(&B.xf_kv[sl]);
      return true;
    };
    auto do_q = [&](uint32_t t) -> bool {
      const uint32_t sl = t & 1u;
      if (!tcu::wait_warp(&B.full_q[sl], (t >> 1) & 1u, abort_flag, err, SITE_TC_TRANSFORM, t)) return false;
      xf_tile(sbase + OFF_Q + sl * kTileBytes, kTile, silu, wt);
      fence_proxy_async_smem();
      mbar_arrive(&B.xf_q[sl]);
      return true;
    };
    for (; it.valid; blk_next<tpb>(p, it, wk)) {
      int vr0, vr1;
      const int n = blk_tiles<tpb>(it, vr0, vr1);
      if (!do_k(ot, vr0) || !do_q(ot)) break;
      if (n > 1 && (!do_q(ot + 1) || !do_k(ot + 1, vr1))) break;
      ot += n;
    }
  }
  // ------------------------------------------------------------------------------------
  // Warps 4-7 (one per TMEM lane quarter; thread r owns row r of every TMEM tile):
  //  * score conversion (fp32 -> masked bf16 in place), job by job;
  //  * the state: S0 into TMEM and the bf16 snapshot at a sequence start; after each
  //    block's state update, S_b once: into the snapshot for the next block's inter
  //    products, or to state_out after the sequence's last block;
  //  * norm modes: each tile's sums of squares over the head's 128 columns of a row, added
  //    into the fp64 per-token total, then one arrival per warp on the tile's counter.
  // Per block: conversions A and B, the sums of tile 0, conversion C, the state, the sums of
  // tile 1 -- the order in which the MMA warp makes them ready.
  // ------------------------------------------------------------------------------------
  else if (warp >= kConvWarp0 && warp < kConvWarp0 + 4) {
    const int r = tid - 32 * kConvWarp0;           // TMEM lane: row of a tile, or d_k row of S
    const uint32_t lane_off = static_cast<uint32_t>(r & ~31) << 16;
    const uint32_t tP = tmem + lane_off + TM_P;
    const uint32_t tS = tmem + lane_off + TM_S;
    const uint32_t snap = sbase + OFF_SNAP;
    const bool skip_publish = (err->inject == INJECT_SKIP_PUBLISH) && blockIdx.x == 0;
    uint32_t jb = 0, nb = 0, ot = 0;
    bool ok = true;
    auto conv = [&](int ncols, bool diag) -> bool {
      if (!tcu::wait_warp(&B.p_full, jb & 1u, abort_flag, err, SITE_TC_CONVERT, jb)) return false;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < ncols / 16; ++c) {
        uint32_t x[16];
        tmem_ld16(tP + 16 * c, x);
        tmem_ld_wait();
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j = 16 * c + 2 * e;
          float a = __uint_as_float(x[2 * e]), b = __uint_as_float(x[2 * e + 1]);
          if (diag) {   // keys up to the query row
            a = (j <= r) ? a : 0.f;
            b = (j + 1 <= r) ? b : 0.f;
          }
          pk[e] = pack_bf16x2(a, b);
        }
        tmem_st8(tP + 8 * c, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&B.p_conv);
      ++jb;
      return true;
    };
    // Sum of squares of row r of own tile t (tile i of sequence s, rows from row0).
    auto publish = [&](uint32_t t, const BlkIter& bi, int u, int vr) -> bool {
      const uint32_t sa = t & 1u;
      if (!tcu::wait_warp(&B.o_full[sa], (t >> 1) & 1u, abort_flag, err, SITE_TC_EPILOGUE, t)) return false;
      tc_fence_after();
      float ss = 0.f;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t x[16];
        tmem_ld16(tmem + lane_off + TM_O + 128 * sa + 16 * c, x);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) ss = fmaf(__uint_as_float(x[e]), __uint_as_float(x[e]), ss);
      }
      tc_fence_before();
      const int i = bi.jb * tpb + u;
      if (r < vr) tcu::red_add_f64(p.ss + bi.row0 + static_cast<int64_t>(i) * kTile + r, static_cast<double>(ss));
      tcu::fence_acq_rel_gpu();
      __syncwarp();
      if ((r & 31) == 0 && !skip_publish)
        tcu::red_add_relaxed_u32(p.cnt + static_cast<int64_t>(bi.s) * p.max_tiles + i, 1u);
      return true;
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
      else if (p.chunk_div > 1) {
        if (s % p.chunk_div != p.chunk_div - 1) return -1;
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
      const int n = blk_tiles<tpb>(it, vr0, vr1);
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
      if (!conv(pad_rows(vr0), true)) break;
      if (n > 1 && !conv(128, false)) break;
      if (norm && !publish(ot, it, 0, vr0)) break;
      if (n > 1 && !conv(pad_rows(vr1), true)) break;
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
      if (norm && n > 1 && !publish(ot + 1, it, 1, vr1)) break;
      ot += n;
    }
  }
  // ------------------------------------------------------------------------------------
  // Warps 16-23: output stores.  Warp e owns TMEM lane quarter e % 4 (32 rows of every
  // tile) and columns 64 * (e / 4 - 4) .. +63 of the head.  Raw mode stores y.  The norm
  // modes wait until every head has published the tile's sums, then store
  // o = bf16(y w) rsqrt(mean(y^2) + eps) [sigmoid(g)], 32 bytes per access; the
  // accumulator is freed after its last read.
  // ------------------------------------------------------------------------------------
  else if (warp >= kEpiWarp0) {
    const int q = warp & 3;
    const int half = (warp - kEpiWarp0) >> 2;
    const int rr = 32 * q + lane;                     // row of the tile
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    const int64_t HD = static_cast<int64_t>(p.H) * kD;
    const float inv_hd = 1.0f / static_cast<float>(HD);
    const int col0 = h * kD + 64 * half;
    uint32_t ot = 0;
    bool ok = true;
    BlkIter it;
    blk_first<tpb>(p, it, wk);
    for (; it.valid && ok; blk_next<tpb>(p, it, wk)) {
      int vr0, vr1;
      const int n = blk_tiles<tpb>(it, vr0, vr1);
      for (int u = 0; u < n && ok; ++u, ++ot) {
        const uint32_t sa = ot & 1u;
        const int i = it.jb * tpb + u;                 // tile of the sequence
        const int vr = u == 0 ? vr0 : vr1;
        const int64_t row = it.row0 + static_cast<int64_t>(i) * kTile + rr;
        const bool valid = rr < vr;
        uint16_t* dst = p.out + row * HD + col0;
        const uint32_t oacc = tmem + lane_off + TM_O + 128 * sa + 64 * half;
        float rn = 1.f;
        uint32_t g0[8], g1[8];   // gate values of columns 0..15 and 16..31 of the current 32
        if (norm) {
          const uint16_t* gsrc = p.g + row * HD + col0;
          if (gate && valid) {   // in flight during the waits
            tcu::ld_nc_v8(gsrc, g0);
            tcu::ld_nc_v8(gsrc + 16, g1);
          }
          unsigned int* cnt = p.cnt + static_cast<int64_t>(it.s) * p.max_tiles + i;
          int go = 1;
          if (lane == 0 && ld_acquire_gpu(cnt) < W)
            go = tcu::poll_count(cnt, W, abort_flag, err, static_cast<uint32_t>(it.s * p.max_tiles + i)) ? 1 : 0;
          if (!__shfl_sync(0xFFFFFFFFu, go, 0)) {
            ok = false;
            break;
          }
          (void)ld_acquire_gpu(cnt);
          if (valid) rn = 1.0f / sqrtf(static_cast<float>(tcu::ld_cg_f64(p.ss + row)) * inv_hd + p.eps);
        }
        // The counter covers the accumulator's completion (its publisher waited for it); the
        // wait here orders this warp's TMEM reads after the MMAs.
        if (!tcu::wait_warp(&B.o_full[sa], (ot >> 1) & 1u, abort_flag, err, SITE_TC_EPILOGUE, ot)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {   // 16 columns at a time
          if (gate && valid && c == 2) {
            tcu::ld_nc_v8(p.g + row * HD + col0 + 32, g0);
            tcu::ld_nc_v8(p.g + row * HD + col0 + 48, g1);
          }
          uint32_t x[16];
          tmem_ld16(oacc + 16 * c, x);
          tmem_ld_wait();
          if (c == 3) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&B.o_empty[sa]);
          }
          uint32_t o[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int col = 64 * half + 16 * c + 2 * e;
            float a = __uint_as_float(x[2 * e]), b = __uint_as_float(x[2 * e + 1]);
            if (norm) {
              // z = bf16(y w): the unnormalised output is rounded before the scale
              const uint32_t zz = pack_bf16x2(a * B.w[col], b * B.w[col + 1]);
              a = __uint_as_float(zz << 16) * rn;
              b = __uint_as_float(zz & 0xFFFF0000u) * rn;
              if (gate) {
                const uint32_t gg = (c & 1) ? g1[e] : g0[e];
                a *= sigmoid_fast(__uint_as_float(gg << 16));
                b *= sigmoid_fast(__uint_as_float(gg & 0xFFFF0000u));
              }
            }
            o[e] = pack_bf16x2(a, b);
          }
          if (valid) tcu::st_na_v8(dst + 16 * c, o);
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
PairKernel pair_kernel(int mode, int C) {
  static const PairKernel k[3][2] = {
      {lightning_prefill_pair_kernel<LA_OUT_RAW, 128>, lightning_prefill_pair_kernel<LA_OUT_RAW, 256>},
      {lightning_prefill_pair_kernel<LA_OUT_RMSNORM, 128>, lightning_prefill_pair_kernel<LA_OUT_RMSNORM, 256>},
      {lightning_prefill_pair_kernel<LA_OUT_RMSNORM_GATE, 128>,
       lightning_prefill_pair_kernel<LA_OUT_RMSNORM_GATE, 256>}};
  return k[mode == LA_OUT_RAW ? 0 : (mode == LA_OUT_RMSNORM ? 1 : 2)][C == 256 ? 1 : 0];
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
    PairKernel kern = pair_kernel(LA_OUT_RMSNORM_GATE, 256);
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
  return up256(sizeof(unsigned int) * static_cast<size_t>(nseq) * (max_tiles ? max_tiles : 1)) +
         up256(sizeof(double) * static_cast<size_t>(tokens > 0 ? tokens : 1)) +
         up256(sizeof(int) * static_cast<size_t>(nseq)) + up256(sizeof(int) * (nw + 1));
}

cudaError_t launch_pair_prefill(const TcArgs& a, cudaStream_t stream) {
  if (a.reverse || a.D != kD || (a.C != 128 && a.C != 256)) return cudaErrorInvalidValue;
  const int max_tiles = (a.max_len + kTile - 1) / kTile;
  const size_t cnt_bytes = up256(sizeof(unsigned int) * static_cast<size_t>(a.nseq) * (max_tiles ? max_tiles : 1));
  const size_t ss_bytes = up256(sizeof(double) * static_cast<size_t>(a.tokens > 0 ? a.tokens : 1));
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
  // Packed batches of several sequences: the longest-first worker plan.
  if (a.cu && a.nseq > 1 && a.nseq <= kPlanMaxSeqs && nw <= 256) {
    int* sched = reinterpret_cast<int*>(a.ws + cnt_bytes + ss_bytes);
    int* wstart = reinterpret_cast<int*>(a.ws + cnt_bytes + ss_bytes + sched_bytes);
    plan_kernel<<<1, kPlanThreads, 0, stream>>>(a.cu, a.nseq, nw, a.skip_single, sched, wstart);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    p.sched = sched;
    p.wstart = wstart;
  }
  const PairKernel kernel = pair_kernel(a.mode, a.C);
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
