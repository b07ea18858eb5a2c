// Lightning Attention prefill on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// What is computed ("六十四：MiniMax-01", section 3; "MiniMax-Text-01 405B MoE模型架构与
// 训练策略解析", section 2.1; "MiniMax-01技术报告解读（二）计算优化", section 3):
// causal linear attention with phi = SiLU on q and k, evaluated block by block with the
// block size C (256 in the deployment config).  For block j with rows Q_j, K_j, V_j:
//     O_j = (phi(Q_j) phi(K_j)^T (.) M) V_j + phi(Q_j) S_{j-1}          (intra + inter)
//     S_j = S_{j-1} + phi(K_j)^T V_j                                    (fp32 state carry)
// followed by o = RMSNorm over the H*D head concatenation of a token times sigmoid(g).
//
// Design (B200, sm_100a):
//  * One CTA owns one (head, 64-column slice of d_v) chain and walks all sequences of its
//    group.  With H = 64 that is 128 CTAs, one per SM, all resident at once, and one group;
//    with fewer heads several groups of CTA pairs split the sequences between them.
//  * Work is tiled in 128-row tiles (the tcgen05 M).  C = 256 is two tiles per block: the
//    second tile multiplies by the first tile's keys densely and by its own keys under the
//    causal mask; the all-zero upper-right quarter of the 256 x 256 block is never issued.
//  * The two CTAs of a head form a cluster.  Each loads (TMA, 128-byte swizzle) its own
//    64-column box of the Q and K tiles plus its V slice, applies SiLU (packed bf16x2
//    arithmetic) to its boxes with six transform warps, and writes the result both into its own shared memory and into
//    its partner's (distributed shared memory), so each SiLU is computed once per head and
//    both CTAs end up with the full phi(Q), phi(K) tiles.  Q tiles use a two-slot ring and
//    K/V tiles a three-slot ring, so the next block's first tile loads while the second
//    tile of a 256-block still reads the first tile's keys and values.  The gate tile is
//    only prefetched into L2.
//  * One thread issues all MMAs (bf16 in, fp32 accumulate in TMEM), per tile:
//      P   = phi(Q) phi(K)^T          SS, M128 x N(<=128) x K128, into TMEM
//      O   = P_bf16 V                 TS (P read back from TMEM), M128 x N64 x K(<=128)
//      O  += phi(Q) S_snap            SS, M128 x N64 x K128 (S_snap = bf16 copy of S)
//      S  += phi(K)^T V               SS (both operands MN-major), M128 x N64 x K(<=128)
//    The fp32 state S stays in TMEM for the whole sequence; the inter product comes last
//    so the snapshot of S taken at the previous block end is ready by then.
//    Score tiles alternate between two TMEM regions so that P of the next key/query tile
//    is computed while the current one is being converted.
//  * A conversion warpgroup turns P (fp32, TMEM) into masked bf16 in place.
//  * The kernel is instantiated per output mode and block size.  The epilogue reader
//    warpgroup owns the state (S0 in, the bf16 snapshot of S at each block end, the final
//    state out) and reads O once, releasing the accumulator at once.  In the raw mode it
//    stores y directly.  In the norm modes it parks z = y * w as bf16 pairs in two spare
//    TMEM tiles, adds each row's sum of squares into an fp64 per-token accumulator in
//    global memory (red.add; the fp64 sum of the fp32 partials is exact whenever a token's
//    partials span less than 2^22, so the result does not depend on the order the
//    additions land in) and bumps the tile's arrival counter (at a block end only after
//    the state snapshot is out, since the release waits for the additions).  Four storer warps, one per TMEM lane quarter, load their rows of the
//    gate, wait until all H * 2 CTAs have arrived for the tile (the gate loads are in
//    flight meanwhile), scale z by rsqrt(mean(y^2) + eps) * sigmoid(g) in registers and
//    store each row's 128 bytes straight from registers.
//  * Every wait is bounded (globaltimer); a wait that runs out records LA_ERR_TIMEOUT in
//    the workspace and the CTA drains its async work, frees TMEM and exits.
//  * Reverse time (raw mode, for the backward's sums over t >= i): each sequence's
//    128-row tiles are walked from the last to the first and the diagonal tile keeps the
//    keys at or after the query row.  The rows inside a tile keep their order, so the
//    partial tile (now the first one walked) has its valid rows on top as before, and the
//    block pairs simply start at the sequence end.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "la_common.cuh"
#include "la_prefill_tc.h"
#include "la_sm100.cuh"
#include "la_tc_util.cuh"

namespace la {
using namespace sm100;

namespace {

constexpr int kD = 128;          // head dim (d_k = d_v)
constexpr int kDV = 64;          // d_v slice per CTA
constexpr int kNdv = kD / kDV;   // CTAs per head
constexpr int kTile = 128;       // rows per tile (MMA M)
constexpr int kThreads = 640;    // 20 warps
constexpr int kXfWarp0 = 2;      // transform warps 2..7
constexpr int kXfThreads = 192;
constexpr int kNQ = 2;           // Q slots
constexpr int kNKV = 3;          // K / V slots (a 256-block's first tile stays while the next loads)
constexpr int kReadWarp0 = 12;   // epilogue readers: warps 12..15 (TMEM lane quarters 0..3)
constexpr int kStoreWarp0 = 16;  // epilogue storers: warps 16..19 (TMEM lane quarters 0..3)
constexpr int kQuarterRows = 32; // rows of a tile one reader / storer warp owns

constexpr uint32_t kQBytes = kTile * kD * 2;     // 32 KiB (two 64-column swizzled boxes)
constexpr uint32_t kKBytes = kQBytes;
constexpr uint32_t kVBytes = kTile * kDV * 2;    // 16 KiB
constexpr uint32_t kSnapBytes = kD * kDV * 2;    // 16 KiB
constexpr uint32_t kBoxBytes = kTile * 64 * 2;   // one 128-row x 64-column box

constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + kNQ * kQBytes;
constexpr uint32_t OFF_V = OFF_K + kNKV * kKBytes;
constexpr uint32_t OFF_SNAP = OFF_V + kNKV * kVBytes;
constexpr uint32_t OFF_BARS = OFF_SNAP + kSnapBytes;

// TMEM columns (512 allocated; 128 lanes each)
constexpr uint32_t TM_S = 0;      // fp32 state slice, 64 columns
constexpr uint32_t TM_O = 64;     // 2 output accumulators x 64 columns
constexpr uint32_t TM_Z = 192;    // 2 parked z tiles x 32 columns (bf16 pairs)
constexpr uint32_t TM_P = 256;    // 2 score tiles x 128 columns
constexpr uint32_t kTmemCols = 512;

struct Bars {
  uint64_t full_q[kNQ], q_empty[kNQ], full_kv[kNKV], kv_empty[kNKV], xformed[kNKV];
  uint64_t p_full[2], p_conv[2], pv_done[2];   // per TMEM score region
  uint64_t o_full[2], o_empty[2];
  uint64_t s_done, snap_ready, final_bar;
  uint64_t z_full[2][4], z_free[2][4];   // per parked-z slot and TMEM lane quarter
  uint32_t tmem_base;
  int abort_flag;
  float w[kDV];
};

constexpr uint32_t kSmemBytes = OFF_BARS + sizeof(Bars) + 1024;  // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct TcParams {
  const float* state_in;
  float* state_out;
  const int* cu;
  int nseq, T, H, C, phi_identity, mode, max_tiles;
  int64_t tokens;
  float eps;
  const float* w;
  const uint16_t* g;   // gate [tokens, H * D] (gated mode)
  ErrRec* err;
  unsigned int* cnt;   // [nseq * max_tiles] arrivals per tile
  double* ss;          // [tokens] sum of squares over the head concatenation
  uint16_t* out;
  const int* state_index;  // optional [nseq]: state slot of each sequence (else the index)
  int skip_single;         // nonzero: one-token sequences belong to a decode step: skip them
  int ngroups;             // sequence groups: the CTA pairs of group g take sequences g, g + G, ...
};

// Shared-memory descriptor templates with start address 0; an operand at shared address a
// is template + ((a >> 4) & 0x3FFF) (the 14-bit start field; adding in-tile offsets to it
// never carries out of the field because every operand lies below 256 KiB).
// Building descriptors this way keeps the single MMA-issuing thread at a few instructions
// per MMA, which is what lets small-N MMAs run at the tensor pipe's rate.
constexpr uint64_t sdesc_template(uint32_t lbo, uint32_t sbo) {
  return (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) | (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) |
         (1ull << 46) | (2ull << 61);
}
constexpr uint64_t kDescK = sdesc_template(16, 1024);          // K-major, 128-byte swizzle
constexpr uint64_t kDescMN = sdesc_template(kBoxBytes, 1024);  // MN-major, 64-element chunks kBoxBytes apart
// Descriptor of the operand at shared address `a`.  Only the low 18 address bits enter
// the 14-bit start field: in a cluster the shared address of a CTA other than rank 0 has
// higher bits set, which must not spill into the leading-byte-offset field.
__device__ __forceinline__ uint64_t desc_at(uint64_t tmpl, uint32_t a) { return tmpl + ((a >> 4) & 0x3FFFu); }

constexpr uint32_t kIdescQS = make_idesc_bf16(128, kDV, 0, 1);
constexpr uint32_t kIdescPV = make_idesc_bf16(128, kDV, 0, 1);
constexpr uint32_t kIdescDS = make_idesc_bf16(128, kDV, 1, 1);

__device__ __forceinline__ int pad_rows(int vr) { return vr <= 32 ? 32 : (vr <= 64 ? 64 : 128); }

// Rows [row0, row0 + L) of sequence s.  Invalid cu_seqlens entries are reported and the
// sequence is treated as empty (every role and every CTA reaches the same decision).
// Returns true for a sequence this call leaves alone entirely (a one-token sequence of a
// mixed step, which the decode kernel handles): L = 0 and its state is not touched.
__device__ __forceinline__ bool seq_range(const TcParams& p, int s, int64_t& row0, int& L) {
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

// The (sequence, tile) order every role walks: this CTA's group's sequences (every
// p.ngroups-th from its group index), empty sequences have no tiles.
struct TileIter {
  int s, i, nt, L;
  int64_t row0;
  bool valid;
};
__device__ __forceinline__ void tile_next(const TcParams& p, TileIter& it) {
  if (it.valid && it.i + 1 < it.nt) {
    ++it.i;
    return;
  }
  for (int s = it.s + p.ngroups; s < p.nseq; s += p.ngroups) {
    int64_t r0;
    int L;
    seq_range(p, s, r0, L);
    const int nt = (L + kTile - 1) / kTile;
    if (nt > 0) {
      it.s = s;
      it.i = 0;
      it.nt = nt;
      it.L = L;
      it.row0 = r0;
      it.valid = true;
      return;
    }
  }
  it.s = p.nseq;
  it.valid = false;
}
__device__ __forceinline__ void tile_first(const TcParams& p, TileIter& it, int grp) {
  it.s = grp - p.ngroups;
  it.i = 0;
  it.nt = 0;
  it.L = 0;
  it.row0 = 0;
  it.valid = false;
  tile_next(p, it);
}

// Bounded wait for phase `parity` of an mbarrier.  Returns false (after recording a
// timeout, or because another role already did) when the CTA is aborting.  The polling
// loop is out of line: only the first test is inlined at each of the many wait sites,
// which keeps the kernel's code (and its instruction-cache footprint) small.
__device__ __noinline__ bool wait_bar_slow(uint64_t* bar, uint32_t parity, int* abort_flag, ErrRec* err,
                                           uint32_t site, uint32_t index) {
  const uint64_t t0 = globaltimer_ns();
  const uint64_t lim = wait_limit_ns(err);
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait_sleep(bar, parity, 20000)) return true;   // suspends: no issue slots used
    if ((n & 3u) == 0) {
      if (*reinterpret_cast<volatile int*>(abort_flag) != 0) return false;
      if (globaltimer_ns() - t0 > lim) {
        report(err, LA_ERR_TIMEOUT, site, index, parity);
        *reinterpret_cast<volatile int*>(abort_flag) = 1;
        return false;
      }
    }
  }
}
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Bars& B, const TcParams& p, uint32_t site,
                                      uint32_t index) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_bar_slow(bar, parity, &B.abort_flag, p.err, site, index);
}

// Bounded poll (one thread) until the arrival count at c reaches W, out of line for the
// same reason; false when the CTA is aborting or the wait ran out (recorded).
__device__ __noinline__ bool poll_count_slow(unsigned int* c, uint32_t W, int* abort_flag, ErrRec* err,
                                             uint32_t index) {
  const uint64_t t0 = globaltimer_ns();
  const uint64_t lim = wait_limit_ns(err);
  for (uint32_t ns = 32; ld_acquire_gpu(c) < W; ns = ns < 256 ? 2 * ns : ns) {
    __nanosleep(ns);
    if (*reinterpret_cast<volatile int*>(abort_flag) != 0) return false;
    if (globaltimer_ns() - t0 > lim) {
      report(err, LA_ERR_TIMEOUT, SITE_TC_NORM_WAIT, index, ld_acquire_gpu(c));
      *reinterpret_cast<volatile int*>(abort_flag) = 1;
      return false;
    }
  }
  return true;
}

// Short bounded wait used while draining at exit (never records an error).
__device__ __noinline__ void drain_bar(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) return;
  }
}

// The same wait taken by every lane of a warp: the outcome is made warp-uniform so that
// the .sync.aligned tcgen05 instructions that follow always see a converged warp.
__device__ __forceinline__ bool wait_bar_warp(uint64_t* bar, uint32_t parity, Bars& B, const TcParams& p,
                                              uint32_t site, uint32_t index) {
  const bool ok = wait_bar(bar, parity, B, p, site, index);
  return __all_sync(0xFFFFFFFFu, ok);
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v);
// Columns 16j .. 16j + 15 of one row of S (fp32 bits) into the bf16 snapshot: two
// 16-byte chunks of the row's 128-byte-swizzled line.
__device__ __forceinline__ void store_snap16(uint32_t snap, int row, int j, const uint32_t (&r)[16]) {
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    const uint32_t* a = r + 8 * h2;
    sts128(snap + sw128_offset(row, 2 * j + h2),
           make_uint4(pack_bf16x2(__uint_as_float(a[0]), __uint_as_float(a[1])),
                      pack_bf16x2(__uint_as_float(a[2]), __uint_as_float(a[3])),
                      pack_bf16x2(__uint_as_float(a[4]), __uint_as_float(a[5])),
                      pack_bf16x2(__uint_as_float(a[6]), __uint_as_float(a[7]))));
  }
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
// Streaming 16-byte store that does not allocate in L1.
__device__ __forceinline__ void st_global_na(uint4* p, uint4 v) {
  asm volatile("st.global.L1::no_allocate.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ double ld_cg_f64(const double* p) {
  double v;
  asm volatile("ld.global.cg.f64 %0, [%1];" : "=d"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_add_release_gpu(unsigned int* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void red_add_f64(double* p, double v) {
  asm volatile("red.relaxed.gpu.global.add.f64 [%0], %1;" ::"l"(p), "d"(v) : "memory");
}

// ======================================================================================
// The kernel
// ======================================================================================
// One instantiation per output mode (la_out_mode) and block size (128 or 256 rows), so
// that each variant's roles compile to straight-line code.
template <int kMode, int kC, bool kRev>
__global__ void __launch_bounds__(kThreads, 1)
lightning_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                            const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw_addr);
  Bars& B = *reinterpret_cast<Bars*>(smem + OFF_BARS);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int h = (blockIdx.x / kNdv) % p.H;
  const int grp = blockIdx.x / (kNdv * p.H);             // sequence group
  const int dvt = static_cast<int>(cluster_ctarank());   // == blockIdx.x % 2 (cluster of 2)
  const uint32_t partner = static_cast<uint32_t>(dvt ^ 1);
  constexpr int tpb = kC / kTile;        // tiles per block (1 or 2)
  constexpr bool norm = kMode != LA_OUT_RAW;
  constexpr bool gate = kMode == LA_OUT_RMSNORM_GATE;
  static_assert(!kRev || kMode == LA_OUT_RAW, "reverse time is a raw-mode variant");
  const int W = p.H * kNdv * 4;          // reader warps contributing to one tile's norm
  // Tile i of a sequence's processing order is physical tile i, or nt - 1 - i when time
  // runs backwards (kRev: the sequence is walked from its end; see the header comment).
  auto phys = [](int i, int nt) { return kRev ? nt - 1 - i : i; };

  if (tid == 0) {
    for (int i = 0; i < kNKV; ++i) {
      mbar_init(&B.full_kv[i], 1);
      mbar_init(&B.xformed[i], 2 * kXfThreads);   // both CTAs' transform threads
      mbar_init(&B.kv_empty[i], 2);               // both CTAs' MMAs released the slot
    }
    for (int i = 0; i < kNQ; ++i) {
      mbar_init(&B.full_q[i], 1);
      mbar_init(&B.q_empty[i], 2);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&B.o_full[i], 1);
      mbar_init(&B.o_empty[i], 128);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&B.p_full[i], 1);
      mbar_init(&B.p_conv[i], 128);
      mbar_init(&B.pv_done[i], 1);
    }
    mbar_init(&B.s_done, 1);
    mbar_init(&B.snap_ready, 128);
    mbar_init(&B.final_bar, 1);
    for (int i = 0; i < 2; ++i)
      for (int q = 0; q < 4; ++q) {
        mbar_init(&B.z_full[i][q], 32);
        mbar_init(&B.z_free[i][q], 32);
      }
    B.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc<kTmemCols>(&B.tmem_base);
  if (tid >= 32 * kReadWarp0 && tid < 32 * kReadWarp0 + kDV)
    B.w[tid - 32 * kReadWarp0] = p.w ? p.w[h * kD + dvt * kDV + (tid - 32 * kReadWarp0)] : 1.0f;
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the partner may arrive on these barriers from now on
  tc_fence_after();
  const uint32_t tmem = B.tmem_base;

  // ------------------------------------------------------------------------------------
  // Warp 0: TMA producers.  Lane 0 streams this CTA's 64-column Q boxes into Q slot
  // t % 2; lane 1 streams its K boxes and V slices into K/V slot t % 3 and prefetches the
  // gate tile into L2 (the storers load their rows of it straight from global memory).
  // The partner CTA supplies the other box of Q and K.  The two rings run independently,
  // so keys and values run ahead of the queries whenever their slots free up earlier.
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
      const int nslots = is_q ? kNQ : kNKV;
      uint32_t uses[kNKV] = {0, 0, 0};
      int t = 0;
      bool ok = true;
      for (int s = grp; s < p.nseq && ok; s += p.ngroups) {
        int64_t row0;
        int L;
        seq_range(p, s, row0, L);
        const int nt = (L + kTile - 1) / kTile;
        for (int i = 0; i < nt; ++i) {
          const int sl = t % nslots;
          uint64_t* empty = is_q ? &B.q_empty[sl] : &B.kv_empty[sl];
          if (uses[sl] > 0 && !wait_bar(empty, (uses[sl] - 1) & 1, B, p, SITE_TC_PRODUCER, t)) {
            ok = false;
            break;
          }
          const int32_t row = static_cast<int32_t>(row0 + static_cast<int64_t>(phys(i, nt)) * kTile);
          if (is_q) {
            mbar_arrive_expect_tx(&B.full_q[sl], kBoxBytes);
            tma_load_2d(smem + OFF_Q + sl * kQBytes + dvt * kBoxBytes, &tm_q, h * kD + dvt * 64, row, &B.full_q[sl],
                        pol);
          } else {
            mbar_arrive_expect_tx(&B.full_kv[sl], kBoxBytes + kVBytes);
            tma_load_2d(smem + OFF_K + sl * kKBytes + dvt * kBoxBytes, &tm_k, h * kD + dvt * 64, row, &B.full_kv[sl],
                        pol);
            tma_load_2d(smem + OFF_V + sl * kVBytes, &tm_v, h * kD + dvt * kDV, row, &B.full_kv[sl], pol);
            if (gate) tma_prefetch_l2_2d(&tm_g, h * kD + dvt * kDV, row);
          }
          uses[sl]++;
          ++t;
        }
      }
      // Drain: every issued load must have landed before the CTA may exit.
      for (int i = 0; i < nslots; ++i)
        if (uses[i] > 0) drain_bar(is_q ? &B.full_q[i] : &B.full_kv[i], (uses[i] - 1) & 1);
    }
  }
  // ------------------------------------------------------------------------------------
  // Warp 1: MMA issuer (one thread).  Score tiles ("jobs": one per query tile and key
  // tile of its block) alternate between two TMEM regions; P of the next job is issued
  // while the conversion warps still work on the current one, so the tensor core is not
  // idle while scores are converted.
  // ------------------------------------------------------------------------------------
  else if (warp == 1) {
    if (lane == 0) {
      uint32_t snap_waits = 0;
      uint32_t k = 0;                  // next job to consume (PV)
      uint32_t kp = 0;                 // next job whose P is issued
      int xf_tile = -1;                // last tile whose transformed data was waited for
      int t = 0;
      bool ok = true;
      TileIter cur, nxt;
      tile_first(p, cur, grp);
      nxt = cur;
      tile_next(p, nxt);

      // Wait (blocking) or test (non-blocking) for the transformed data of tile tt.
      auto take_xf = [&](int tt, bool block) -> int {
        if (xf_tile >= tt) return 1;
        uint64_t* bar = &B.xformed[tt % kNKV];
        const uint32_t par = static_cast<uint32_t>(tt / kNKV) & 1u;
        if (block) {
          if (!wait_bar(bar, par, B, p, SITE_TC_MMA, tt)) return -1;
        } else if (!mbar_try_wait(bar, par)) {
          return 0;
        }
        xf_tile = tt;
        tc_fence_after();
        return 1;
      };
      // K/V slot of key tile kt of the block that tile tt (position u in it) belongs to.
      auto kv_slot = [&](int tt, int u, int kt) { return (kt == u ? tt : tt - 1) % kNKV; };
      // P of job `job` = (tile it / tt, key tile kt) into region job & 1.
      auto issue_p = [&](const TileIter& it, int tt, int kt, uint32_t job) -> bool {
        const uint32_t r = job & 1u;
        if (job >= 2) {
          if (!wait_bar(&B.pv_done[r], ((job - 2) >> 1) & 1, B, p, SITE_TC_MMA, tt)) return false;
          tc_fence_after();
        }
        const int u = it.i % tpb;
        const int vr = min(kTile, it.L - phys(it.i, it.nt) * kTile);
        const uint32_t n = (kt == u) ? static_cast<uint32_t>(pad_rows(vr)) : 128u;
        const uint64_t qd = desc_at(kDescK, sbase + OFF_Q + (tt % kNQ) * kQBytes);
        const uint64_t kd = desc_at(kDescK, sbase + OFF_K + kv_slot(tt, u, kt) * kKBytes);
        const uint32_t idesc = make_idesc_bf16(128, n, 0, 0);
        const uint32_t dst = tmem + TM_P + 128 * r;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4);
          mma_ss(dst, qd + off, kd + off, idesc, kk > 0);
        }
        mma_commit(&B.p_full[r]);
        return true;
      };

      while (ok && cur.valid) {
        const int u = cur.i % tpb;
        const int qs = t % kNQ, ks = t % kNKV;
        const int ob = t & 1;
        const int vr = min(kTile, cur.L - phys(cur.i, cur.nt) * kTile);
        const int nk = pad_rows(vr);
        const uint32_t k0 = k;
        if (kp == k0) {  // P of this tile's first job was not issued ahead
          if (take_xf(t, true) < 0 || !issue_p(cur, t, 0, kp)) { ok = false; break; }
          ++kp;
        }
        const uint32_t od = tmem + TM_O + kDV * ob;
        for (int kt = 0; kt <= u && ok; ++kt) {
          // Issue the next job's P ahead: the next key tile of this tile, or the first
          // job of the next tile if its data is already transformed.
          if (kp == k + 1) {
            if (kt < u) {
              if (!issue_p(cur, t, kt + 1, kp)) { ok = false; break; }
              ++kp;
            } else if (nxt.valid) {
              const int got = take_xf(t + 1, false);
              if (got > 0) {
                if (!issue_p(nxt, t + 1, 0, kp)) { ok = false; break; }
                ++kp;
              }
            }
          }
          if (kt == 0 && t >= 2) {
            if (!wait_bar(&B.o_empty[ob], ((t >> 1) - 1) & 1, B, p, SITE_TC_MMA, t)) { ok = false; break; }
            tc_fence_after();
          }
          const uint32_t r = k & 1u;
          if (!wait_bar(&B.p_conv[r], (k >> 1) & 1, B, p, SITE_TC_MMA, t)) { ok = false; break; }
          tc_fence_after();
          // O (+)= P_bf16 V over this key tile
          const int ksteps = ((kt == u) ? nk : 128) / 16;
          const uint64_t vd = desc_at(kDescMN, sbase + OFF_V + kv_slot(t, u, kt) * kVBytes);
          const uint32_t pa = tmem + TM_P + 128 * r;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            if (kk < ksteps) mma_ts(od, pa + 8 * kk, vd + 128 * kk, kIdescPV, (kt > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&B.pv_done[r]);
          // The first tile's keys and values of a 256-block have no reader after this.
          // Slot releases go to both CTAs: the partner writes its transformed boxes here.
          if (kt < u) mma_commit_multicast(&B.kv_empty[kv_slot(t, u, kt)], 0x3);
          ++k;
        }
        if (!ok) break;
        // O += phi(Q) S_snap
        if (u == 0) {
          if (!wait_bar(&B.snap_ready, snap_waits & 1, B, p, SITE_TC_MMA, t)) { ok = false; break; }
          snap_waits++;
          tc_fence_after();
        }
        {
          const uint64_t qd = desc_at(kDescK, sbase + OFF_Q + qs * kQBytes);
          const uint64_t sd = desc_at(kDescMN, sbase + OFF_SNAP);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(od, qd + static_cast<uint64_t>(((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4), sd + 128 * kk,
                   kIdescQS, 1);
        }
        mma_commit(&B.o_full[ob]);
        mma_commit_multicast(&B.q_empty[qs], 0x3);   // phi(Q) of this tile has no reader after this
        // S += phi(K)^T V
        {
          const uint64_t kd = desc_at(kDescMN, sbase + OFF_K + ks * kKBytes);
          const uint64_t vd = desc_at(kDescMN, sbase + OFF_V + ks * kVBytes);
          const int ksteps = nk / 16;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            if (kk < ksteps) mma_ss(tmem + TM_S, kd + 128 * kk, vd + 128 * kk, kIdescDS, 1);
        }
        const bool blk_end = (u == tpb - 1) || (cur.i == cur.nt - 1);
        // This tile's keys and values are done unless the second tile of its block follows.
        if (blk_end) mma_commit_multicast(&B.kv_empty[ks], 0x3);
        if (blk_end) mma_commit(&B.s_done);
        ++t;
        cur = nxt;
        tile_next(p, nxt);
      }
      // Drain: all MMAs complete before TMEM is released.
      mma_commit(&B.final_bar);
      drain_bar(&B.final_bar, 0);
    }
  }
  // ------------------------------------------------------------------------------------
  // Warps 2-7: SiLU of this CTA's Q and K boxes, written to both CTAs of the pair; zero
  // tail rows of K (both copies) and of this CTA's V slice.  Keys are transformed as soon
  // as they land (one tile ahead when possible), so only the query box stands between a
  // query slot's load and the MMAs that free it.
  // ------------------------------------------------------------------------------------
  else if (warp >= kXfWarp0 && warp < kXfWarp0 + kXfThreads / 32) {
    const int wt = tid - 32 * kXfWarp0;
    constexpr int kBoxChunks = static_cast<int>(kBoxBytes / 16);   // 16 bytes = 8 bf16
    // The partner's shared window maps this CTA's offsets one to one.
    const uint32_t remote = mapa_shared(sbase, partner);
    // SiLU of one 128 x 64 box in place, mirrored into the partner; rows >= zero_from are
    // zeroed instead.  Four chunks per thread are loaded before any is stored.
    auto xf_box = [&](uint32_t off0, int zero_from) {
      for (int c0 = wt; c0 < kBoxChunks; c0 += 4 * kXfThreads) {
        uint4 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int c = c0 + j * kXfThreads;
          v[j] = (c < kBoxChunks) ? lds128(sbase + off0 + 16u * c) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int c = c0 + j * kXfThreads;
          if (c < kBoxChunks) {
            uint4 x = v[j];
            if ((c >> 3) >= zero_from) {
              x = make_uint4(0, 0, 0, 0);
            } else if (!p.phi_identity) {
              x = tcu::silu8(x);
            }
            sts128(sbase + off0 + 16u * c, x);
            st_cluster128(remote + off0 + 16u * c, x);
          }
        }
      }
    };
    // Keys (and the zeroed tail of the values) of tile tt.
    auto xf_keys = [&](const TileIter& it, int tt) {
      const int ks = tt % kNKV;
      const int vr = min(kTile, it.L - phys(it.i, it.nt) * kTile);
      xf_box(OFF_K + ks * kKBytes + dvt * kBoxBytes, vr);
      if (vr < kTile) {
        const uint32_t va = sbase + OFF_V + ks * kVBytes;
        for (int c = wt; c < static_cast<int>(kVBytes / 16); c += kXfThreads)
          if ((c >> 3) >= vr) sts128(va + 16u * c, make_uint4(0, 0, 0, 0));
      }
    };
    TileIter cur, nxt;
    tile_first(p, cur, grp);
    nxt = cur;
    tile_next(p, nxt);
    int t = 0;
    int k_done = -1;   // last tile whose keys this thread has transformed
    while (cur.valid) {
      const int qs = t % kNQ, ks = t % kNKV;
      if (k_done < t) {
        if (!wait_bar_warp(&B.full_kv[ks], (t / kNKV) & 1, B, p, SITE_TC_TRANSFORM, t)) break;
        xf_keys(cur, t);
        k_done = t;
      }
      if (!wait_bar_warp(&B.full_q[qs], (t / kNQ) & 1, B, p, SITE_TC_TRANSFORM, t)) break;
      xf_box(OFF_Q + qs * kQBytes + dvt * kBoxBytes, kTile);
      // Local and remote writes become visible to both tensor cores before the arrivals.
      fence_proxy_async_cluster();
      mbar_arrive(&B.xformed[ks]);
      mbar_arrive_cluster(mapa_shared(smem_u32(&B.xformed[ks]), partner));
      // The next tile's keys, if they have landed already.
      if (nxt.valid &&
          __all_sync(0xFFFFFFFFu, mbar_test_wait(&B.full_kv[(t + 1) % kNKV], ((t + 1) / kNKV) & 1))) {
        xf_keys(nxt, t + 1);
        k_done = t + 1;
      }
      ++t;
      cur = nxt;
      tile_next(p, nxt);
    }
  }
  // ------------------------------------------------------------------------------------
  // Warps 8-11: score conversion (fp32 -> masked bf16, in place in TMEM), job by job.
  // ------------------------------------------------------------------------------------
  else if (warp >= 8 && warp < 12) {
    const int wt = tid - 256;                      // TMEM lane = row
    const uint32_t lane_off = static_cast<uint32_t>(wt & ~31) << 16;
    uint32_t k = 0;
    bool ok = true;
    for (int s = grp; s < p.nseq && ok; s += p.ngroups) {
      int64_t row0;
      int L;
      seq_range(p, s, row0, L);
      const int nt = (L + kTile - 1) / kTile;
      for (int i = 0; i < nt && ok; ++i) {
        const int u = i % tpb;
        const int vr = min(kTile, L - phys(i, nt) * kTile);
        const int nk = pad_rows(vr);
        for (int kt = 0; kt <= u; ++kt, ++k) {
          const uint32_t r = k & 1u;
          if (!wait_bar_warp(&B.p_full[r], (k >> 1) & 1, B, p, SITE_TC_CONVERT, k)) { ok = false; break; }
          tc_fence_after();
          const bool diag = (kt == u);
          const int ncols = diag ? nk : 128;
          const uint32_t base = tmem + lane_off + TM_P + 128 * r;
          for (int c = 0; c < ncols / 32; ++c) {
            uint32_t x[32];
            tmem_ld32(base + 32 * c, x);
            tmem_ld_wait();
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int j = 32 * c + 2 * e;
              float a = __uint_as_float(x[2 * e]), b = __uint_as_float(x[2 * e + 1]);
              if (diag) {   // keys up to the query row; from it on when time runs backwards
                a = (kRev ? j >= wt : j <= wt) ? a : 0.f;
                b = (kRev ? j + 1 >= wt : j + 1 <= wt) ? b : 0.f;
              }
              pk[e] = pack_bf16x2(a, b);
            }
            tmem_st16(base + 16 * c, pk);
          }
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&B.p_conv[r]);
        }
      }
    }
  }
  // ------------------------------------------------------------------------------------
  // Warps 12-15: epilogue readers.  Read O once, release the TMEM accumulator, add the
  // rows' sums of squares into the fp64 per-token totals, park z = y * w.
  // They also own the state: S0 into TMEM at each sequence start, the bf16 snapshot of S
  // at each block end, and the final state.
  // ------------------------------------------------------------------------------------
  else if (warp >= kReadWarp0 && warp < kStoreWarp0) {
    const int wt = tid - 32 * kReadWarp0;          // TMEM lane = row of the tile / of S
    const int q = warp - kReadWarp0;               // lane quarter
    const uint32_t lane_off = static_cast<uint32_t>(wt & ~31) << 16;
    const uint32_t snap = sbase + OFF_SNAP;
    const int64_t HD = static_cast<int64_t>(p.H) * kD;
    const bool skip_publish = (p.err->inject == INJECT_SKIP_PUBLISH) && blockIdx.x == 0;
    bool ok = true;
    int t = 0;
    uint32_t blk = 0;
    for (int s = grp; s < p.nseq && ok; s += p.ngroups) {
      int64_t row0;
      int L;
      if (seq_range(p, s, row0, L)) continue;   // a one-token sequence of a mixed step
      const int nt = (L + kTile - 1) / kTile;
      // Initial state: S0 (or zeros) into TMEM and the bf16 snapshot.
      const int64_t slot = p.state_index ? __ldg(p.state_index + s) : s;
      const int64_t st_row = ((slot * p.H + h) * kD + wt) * kD + dvt * kDV;
      {
        // 16 columns at a time: TMEM copy (fp32) and snapshot chunks 2j, 2j + 1 (bf16).
#pragma unroll
        for (int j = 0; j < kDV / 16; ++j) {
          uint32_t r[16];
#pragma unroll
          for (int c = 0; c < 16; c += 4) {
            const float4 x = p.state_in ? *reinterpret_cast<const float4*>(p.state_in + st_row + 16 * j + c)
                                        : make_float4(0, 0, 0, 0);
            r[c] = __float_as_uint(x.x); r[c + 1] = __float_as_uint(x.y);
            r[c + 2] = __float_as_uint(x.z); r[c + 3] = __float_as_uint(x.w);
          }
          if (nt == 0) {
            if (p.state_out)
#pragma unroll
              for (int c = 0; c < 16; c += 4)
                *reinterpret_cast<float4*>(p.state_out + st_row + 16 * j + c) =
                    make_float4(__uint_as_float(r[c]), __uint_as_float(r[c + 1]), __uint_as_float(r[c + 2]),
                                __uint_as_float(r[c + 3]));
            continue;
          }
          tmem_st16(tmem + lane_off + TM_S + 16 * j, r);
          store_snap16(snap, wt, j, r);
        }
        if (nt == 0) continue;
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&B.snap_ready);
      }
      for (int i = 0; i < nt; ++i) {
        const int ob = t & 1;
        const int zs = t & 1;
        const int u = i % tpb;
        const int vr = min(kTile, L - phys(i, nt) * kTile);
        const int64_t row = row0 + static_cast<int64_t>(phys(i, nt)) * kTile;
        if (!wait_bar_warp(&B.o_full[ob], (t >> 1) & 1, B, p, SITE_TC_EPILOGUE, t)) { ok = false; break; }
        if (norm && t >= 2 && !wait_bar_warp(&B.z_free[zs][q], ((t >> 1) - 1) & 1, B, p, SITE_TC_EPILOGUE, t)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // Norm modes: z = y * w, parked as bf16 pairs in TMEM for the storer of this
        // quarter.  Raw mode: y is the output and goes straight from here to global memory.
        // The accumulator goes back to the MMA warp as soon as it has been read.
        float ss = 0.f;
        const uint32_t zt = tmem + lane_off + TM_Z + 32 * zs;
        uint4* zdst = reinterpret_cast<uint4*>(p.out + (row + wt) * HD + h * kD + dvt * kDV);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t zh[16];
#pragma unroll
          for (int sub = 0; sub < 2; ++sub) {
            const int c0 = 32 * half + 16 * sub;   // first column of this group of 16
            uint32_t x[16];
            tmem_ld16(tmem + lane_off + TM_O + kDV * ob + c0, x);
            tmem_ld_wait();
            if (c0 == kDV - 16) {
              tc_fence_before();
              mbar_arrive(&B.o_empty[ob]);
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int col = c0 + 2 * e;
              float a = __uint_as_float(x[2 * e]);
              float b = __uint_as_float(x[2 * e + 1]);
              ss = fmaf(a, a, ss);
              ss = fmaf(b, b, ss);
              if (norm) {
                a *= B.w[col];
                b *= B.w[col + 1];
              }
              zh[8 * sub + e] = pack_bf16x2(a, b);
            }
          }
          if (norm) {
            tmem_st16(zt + 16 * half, zh);
          } else if (wt < vr) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
              zdst[4 * half + c] = make_uint4(zh[4 * c], zh[4 * c + 1], zh[4 * c + 2], zh[4 * c + 3]);
          }
        }
        if (norm) {
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&B.z_full[zs][q]);
        }
        const bool blk_end = (u == tpb - 1 || i == nt - 1);
        if (norm) {
          if (wt < vr) red_add_f64(p.ss + row + wt, static_cast<double>(ss));
          if (!blk_end) {
            __syncwarp();
            // One release per warp orders the warp's additions before the arrival count.
            if (lane == 0 && !skip_publish) red_add_release_gpu(p.cnt + static_cast<int64_t>(s) * p.max_tiles + i, 1u);
          }
        }
        // Block end: snapshot S for the next block's inter product, or emit the final state;
        // the release of this tile's sums waits until the snapshot is out.
        if (blk_end) {
          if (!wait_bar_warp(&B.s_done, blk & 1, B, p, SITE_TC_EPILOGUE, t)) { ok = false; break; }
          blk++;
          tc_fence_after();
          const bool last = (i == nt - 1);
#pragma unroll
          for (int j = 0; j < kDV / 16; ++j) {
            uint32_t r[16];
            tmem_ld16(tmem + lane_off + TM_S + 16 * j, r);
            tmem_ld_wait();
            if (last) {
              if (p.state_out)
#pragma unroll
                for (int c = 0; c < 16; c += 4)
                  *reinterpret_cast<float4*>(p.state_out + st_row + 16 * j + c) =
                      make_float4(__uint_as_float(r[c]), __uint_as_float(r[c + 1]), __uint_as_float(r[c + 2]),
                                  __uint_as_float(r[c + 3]));
            } else {
              store_snap16(snap, wt, j, r);
            }
          }
          if (last) {
            tc_fence_before();
          } else {
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&B.snap_ready);
          }
          if (norm) {
            __syncwarp();
            if (lane == 0 && !skip_publish) red_add_release_gpu(p.cnt + static_cast<int64_t>(s) * p.max_tiles + i, 1u);
          }
        }
        ++t;
      }
    }
  }
  // ------------------------------------------------------------------------------------
  // Warps 16-19 (norm modes): epilogue storers, one per TMEM lane quarter (32 rows of every tile).
  // Load the rows' gate values, read the parked z, wait until every reader warp of every
  // CTA has added its sums for the tile, scale z by rsqrt(mean(y^2) + eps) * sigmoid(g)
  // and store the rows from registers.
  // ------------------------------------------------------------------------------------
  else if (warp >= kStoreWarp0 && norm) {
    const int q = warp - kStoreWarp0;              // == warp % 4: the lane quarter it may access
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    const int64_t HD = static_cast<int64_t>(p.H) * kD;
    const float inv_hd = 1.0f / static_cast<float>(HD);
    bool ok = true;
    int t = 0;
    for (int s = grp; s < p.nseq && ok; s += p.ngroups) {
      int64_t row0;
      int L;
      seq_range(p, s, row0, L);
      const int nt = (L + kTile - 1) / kTile;
      for (int i = 0; i < nt; ++i, ++t) {
        const int zs = t & 1;
        const int vr = min(kTile, L - phys(i, nt) * kTile);
        const int r = kQuarterRows * q + lane;     // row of the tile
        const int64_t row = row0 + static_cast<int64_t>(phys(i, nt)) * kTile;
        // This row's 64 gate values (bf16 pairs), loaded before the waits so that their
        // latency overlaps them; the producer has prefetched the tile into L2.
        uint32_t gq[32];
        if (gate) {
          if (r < vr) {
            const uint4* src = reinterpret_cast<const uint4*>(p.g + (row + r) * HD + h * kD + dvt * kDV);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint4 v = __ldg(src + c);
              gq[4 * c] = v.x; gq[4 * c + 1] = v.y; gq[4 * c + 2] = v.z; gq[4 * c + 3] = v.w;
            }
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) gq[c] = 0;
          }
        }
        if (!wait_bar_warp(&B.z_full[zs][q], (t >> 1) & 1, B, p, SITE_TC_EPILOGUE, t)) { ok = false; break; }
        tc_fence_after();
        uint32_t z[32];
        tmem_ld32(tmem + lane_off + TM_Z + 32 * zs, z);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&B.z_free[zs][q]);
        if (norm) {
          unsigned int* c = p.cnt + static_cast<int64_t>(s) * p.max_tiles + i;
          int go = 1;
          if (lane == 0 && ld_acquire_gpu(c) < static_cast<uint32_t>(W))
            go = poll_count_slow(c, static_cast<uint32_t>(W), &B.abort_flag, p.err,
                                 static_cast<uint32_t>(s * p.max_tiles + i)) ? 1 : 0;
          if (!__shfl_sync(0xFFFFFFFFu, go, 0)) { ok = false; break; }
          (void)ld_acquire_gpu(c);
          const float rn = (r < vr) ? 1.0f / sqrtf(static_cast<float>(ld_cg_f64(p.ss + row + r)) * inv_hd + p.eps) : 0.0f;
          if (gate) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              z[e] = pack_bf16x2(__uint_as_float(z[e] << 16) * (rn * sigmoid_fast(__uint_as_float(gq[e] << 16))),
                                 __uint_as_float(z[e] & 0xFFFF0000u) *
                                     (rn * sigmoid_fast(__uint_as_float(gq[e] & 0xFFFF0000u))));
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              z[e] = pack_bf16x2(__uint_as_float(z[e] << 16) * rn, __uint_as_float(z[e] & 0xFFFF0000u) * rn);
          }
        }
        // Each lane writes its row's 128 contiguous bytes (the 64-column slice of the head).
        if (r < vr) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + (row + r) * HD + h * kD + dvt * kDV);
#pragma unroll
          for (int c = 0; c < 8; ++c) st_global_na(dst + c, make_uint4(z[4 * c], z[4 * c + 1], z[4 * c + 2], z[4 * c + 3]));
        }
      }
    }
  }

  // Teardown: all roles are done (or aborted with their async work drained).  The cluster
  // barrier keeps this CTA's shared memory alive until the partner has stopped writing to
  // it and arriving on its barriers.
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

}  // namespace

// Clusters (head pairs) that fit on the current device at once; cached per device.
int max_active_clusters() {
  static int cache[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    if (cudaFuncSetAttribute(lightning_prefill_tc_kernel<LA_OUT_RMSNORM_GATE, 256, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes)) != cudaSuccess)
      return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kNdv);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kNdv;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, lightning_prefill_tc_kernel<LA_OUT_RMSNORM_GATE, 256, false>, &cfg) !=
        cudaSuccess)
      n = -1;
    cache[dev] = n;
  }
  const int pairs = pair_max_active_clusters();
  return std::min(cache[dev], pairs);
}

bool tc_eligible(const TcShape& s, int num_sms) {
  (void)num_sms;
  if (!s.bf16 || s.D != kD || (s.C != 128 && s.C != 256) || s.H < 1) return false;
  // The cross-head norm exchange needs every head's CTA pair resident at once.
  if (s.mode != LA_OUT_RAW && s.H > max_active_clusters()) return false;
  return true;
}

size_t tc_workspace_bytes(int nseq, int max_len, int64_t tokens, int H, int D, int C) {
  (void)D;
  (void)C;
  const size_t max_tiles = (static_cast<size_t>(max_len) + kTile - 1) / kTile;
  const size_t own = up256(sizeof(unsigned int) * static_cast<size_t>(nseq) * (max_tiles ? max_tiles : 1)) +
                     up256(sizeof(double) * static_cast<size_t>(tokens > 0 ? tokens : 1));
  return std::max(own, pair_workspace_bytes(nseq, max_len, tokens, H));
}

cudaError_t launch_tc_prefill(const TcArgs& a, int num_sms, cudaStream_t stream) {
  (void)num_sms;
  // Both directions of time run on the pair kernel.
  return launch_pair_prefill(a, stream);
  const int max_tiles = (a.max_len + kTile - 1) / kTile;
  const size_t cnt_bytes = up256(sizeof(unsigned int) * static_cast<size_t>(a.nseq) * (max_tiles ? max_tiles : 1));
  const size_t ss_bytes = up256(sizeof(double) * static_cast<size_t>(a.tokens > 0 ? a.tokens : 1));
  TcParams p{};
  p.state_in = a.state_in;
  p.state_out = a.state_out;
  p.cu = a.cu;
  p.nseq = a.nseq;
  p.T = a.T;
  p.H = a.H;
  p.C = a.C;
  p.phi_identity = a.phi_identity;
  p.mode = a.mode;
  p.max_tiles = max_tiles;
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

  const int64_t cols = static_cast<int64_t>(a.H) * kD;
  CUtensorMap mq, mk, mv, mg;
  if (!make_map(&mq, a.q, a.tokens, cols) || !make_map(&mk, a.k, a.tokens, cols) ||
      !make_map(&mv, a.v, a.tokens, cols))
    return cudaErrorInvalidValue;
  if (a.mode == LA_OUT_RMSNORM_GATE) {
    if (!make_map(&mg, a.g, a.tokens, cols)) return cudaErrorInvalidValue;
  } else {
    mg = mq;  // never read
  }
  // Arrival counters and the fp64 sums start at zero on every call.
  cudaError_t e = cudaMemsetAsync(a.ws, 0, cnt_bytes + (a.mode != LA_OUT_RAW ? ss_bytes : 0), stream);
  if (e != cudaSuccess) return e;
  using Kernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, TcParams);
  static const Kernel kernels[3][2] = {
      {lightning_prefill_tc_kernel<LA_OUT_RAW, 128, false>, lightning_prefill_tc_kernel<LA_OUT_RAW, 256, false>},
      {lightning_prefill_tc_kernel<LA_OUT_RMSNORM, 128, false>,
       lightning_prefill_tc_kernel<LA_OUT_RMSNORM, 256, false>},
      {lightning_prefill_tc_kernel<LA_OUT_RMSNORM_GATE, 128, false>,
       lightning_prefill_tc_kernel<LA_OUT_RMSNORM_GATE, 256, false>}};
  // Time running backwards (raw mode only): the backward's reverse-time passes.
  static const Kernel kernels_rev[2] = {lightning_prefill_tc_kernel<LA_OUT_RAW, 128, true>,
                                        lightning_prefill_tc_kernel<LA_OUT_RAW, 256, true>};
  if (a.reverse && a.mode != LA_OUT_RAW) return cudaErrorInvalidValue;
  const Kernel kernel = a.reverse ? kernels_rev[a.C == 256 ? 1 : 0]
                                  : kernels[a.mode == LA_OUT_RAW ? 0 : (a.mode == LA_OUT_RMSNORM ? 1 : 2)]
                                           [a.C == 256 ? 1 : 0];
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  // Sequence groups: with few heads, the CTA pairs of several groups share the sequences
  // (group g takes every G-th), as many as fit on the GPU at once (the norm exchange needs
  // all pairs of a sequence's group resident; all groups together fit in one wave).
  const int maxc = max_active_clusters();
  p.ngroups = maxc > a.H ? std::max(1, std::min(a.nseq, maxc / a.H)) : 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.H * kNdv * p.ngroups);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kNdv;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kernel, mq, mk, mv, mg, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace la
