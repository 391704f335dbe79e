// Tensor-core fused SDPA forward for sm_100a: TMA + tcgen05/TMEM, online
// softmax, in-kernel decomposed rel-pos bias and masks.
//
// softmax(Q.K^T*scale + bias).V without materialising the T_q x T_kv score
// matrix (mlx-examples issue "segment_anything: fuse attention with
// mx.fast.scaled_dot_product_attention": the fused call avoids the 4096x4096
// per-head matrix and the separate softmax pass).  The bias is SAM's
// decomposed relative position (candle PR "SDPA with Relative Positional
// Embeddings": term_h / term_w injected into the scores) or an Axon :mask
// (Axon PR "Add scaled_dot_product_attention", :mask option).
//
// One CTA owns 256 query rows of one (batch, head) as two 128-row tiles A/B
// and streams the K/V tiles of its kv head (hk = h / (Hq/Hkv), Axon PR GQA
// item) through a shared-memory ring.  Warp roles (384 threads):
//   warps 0-3   softmax of tile A (thread = query row = TMEM lane)
//   warps 4-7   softmax of tile B
//   warp  8     TMA producer (Q once, then K_j / V_j per stage)
//   warp  9     TMEM owner and MMA issuer (one elected thread)
//   warps 10-11 idle
// TMEM columns: S_A [0,128), S_B [128,256), O_A [256,256+D), O_B [256+D, 256+2D);
// P (bf16) is the A operand of the P.V MMA straight from TMEM: in its own
// columns at head_dim 64, over the first BN/2 columns of its S tile at 128.
//
// Per KV tile j the MMA warp issues S_t = Q_t.K_j^T (SS, both K-major) and,
// once softmax t has written P_t, O_t += P_t.V_j (TS, V MN-major).  The commit
// that signals "S_t(j+1) ready" also covers O_t += P_t(j).V_j, so softmax t may
// rescale O_t in place when its running max grows.  It does so only when the
// max grows by more than 2^8: every term stays relative to the same (stale)
// max, so the final O/l is unchanged up to rounding.
//
// Rel-pos: before the loop, Ph_t = Q_t.Rh^T and Pw_t = Q_t.Rw^T are computed
// on the tensor cores into TMEM (tables zero-padded to a multiple of 16
// rows), and each thread scatters its row's rel_h[i, kh] = Ph[i, qh - kh + Kh - 1]
// and rel_w[i, kw] = Pw[i, qw - kw + Kw - 1] (times log2 e) into shared
// memory, from where the loop adds them to the scores before the row max.
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "sm100.cuh"
#include "softmax_tile.cuh"
#include "tmap.h"

namespace sdpa {
namespace {

using namespace sm100;

constexpr int kThreads = 384;
constexpr int kMaxSplit = 8;  // parts one unit's key range may be split into
constexpr int kRegsLaunch = 168;   // registers per thread the kernel is launched with
constexpr int kRegsSoftmax = 224;  // after setmaxnreg, softmax warpgroups
constexpr int kRegsOther = 56;     // after setmaxnreg, producer / MMA warpgroup
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther <= kThreads * kRegsLaunch, "register split");
constexpr int kRowsPerTile = 128;
constexpr int kRelHMax = 64;  // key-grid height limit of the tensor-core rel-pos path
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// TC_FLOAT_TMA / TC_BOOL_TMA: the mask tensors of TC_FLOAT / TC_BOOL, 64-key
// tiles brought into shared memory by the producer warp (TMA, two stages per
// query tile) instead of per-row global loads in the softmax warps.
enum TcMask { TC_NONE = 0, TC_RANGE = 1, TC_FLOAT = 2, TC_BOOL = 3, TC_FLOAT_TMA = 4, TC_BOOL_TMA = 5 };

struct TcArgs {
  CUtensorMap tq, tk, tv, trh, trw;
  CUtensorMap tm;  // TC_*_TMA: the mask as (key, query row, head, batch), 64 x 128 boxes
  CUtensorMap to;  // out, 64-column x 32-row boxes: a softmax warp stores its rows by TMA
  void* out;
  long long sob, soh, sot;  // element strides of out (batch, head, token)
  float* lse;
  const void* mask;
  long long msb, msh, msq;
  long long offset, window;
  int B, Hq, Hkv, Tq, Tkv, group;
  int mask_kind;
  float scale_log2;
  int qw_n, kh_n, kw_n;
  int rel_n;  // rows of the padded rel tables (multiple of 16, <= 128)
  int mask_vec;  // mask rows allow 16-byte vector loads
  // Work decomposition over a 1-D grid.  A unit is one 256-row query block of
  // one (batch, head); units are numbered with the query block fastest.  CTAs
  // [0, n_full) each take unit blockIdx.x whole; after them every n_split
  // consecutive CTAs share the key range of one further unit (n_full + i),
  // each taking one contiguous part, merged in-kernel by the last to finish.
  int nqblk;     // query blocks per (batch, head)
  int n_full;    // units taken whole, first in launch order
  int n_split;   // parts per split unit (1 = no split units)
  int reverse_q; // take query blocks last-first (causal: the longest rows start first)
  int head_fast; // number units head-fastest (a mask tensor shared by every head: the heads of a
                 // query block run together and read its mask rows once from DRAM)
  float* ws_o;   // [split units][n_split][D/4][256] float4: unnormalised partial outputs
  float2* ws_ml; // [split units][n_split][256] (running max in log2 units, sum)
  int* ws_cnt;   // [split units] arrival counters, zero between launches
  int* err;
  // the divisors of the unit decode and of the query grid, as FastDiv
  FastDiv fd_split, fd_hq, fd_nqblk, fd_group, fd_qw;
};

template <int D, int BN, int KW, int NS, int MT = 0>  // MT: bytes per mask element (0: no mask tiles)
struct Layout {
  static constexpr int kPanels = D / 64;
  static constexpr int kQBytes = kPanels * kRowsPerTile * 128;  // one Q tile
  static constexpr int kKVBytes = kPanels * BN * 128;           // one K or V tile
  static constexpr int kRelRows = KW > 0 ? kRelHMax + KW : 0;  // rel_h rows then rel_w rows, 256 floats each
  static constexpr int oQ = 0;
  static constexpr int oK = oQ + 2 * kQBytes;
  static constexpr int oV = oK + NS * kKVBytes;
  static constexpr int oRel = oV + NS * kKVBytes;
  static constexpr int kMaskBytes = kRowsPerTile * BN * MT;  // one query tile's mask tile
  static constexpr int oMask = oRel + kRelRows * 256 * 4;            // [query tile][stage]
  static constexpr int oBar = oMask + 4 * kMaskBytes;
  static constexpr int kBars = 4 * NS + 20 + (MT ? 8 : 0);
  static constexpr int kTotal = oBar + kBars * 8 + 32;
  static constexpr int kAlloc = kTotal + 1024;  // slack for 1024-byte alignment
  static_assert(kAlloc <= 232448, "shared memory budget");
  static_assert(KW == 0 || (BN % (KW > 0 ? KW : 1) == 0), "key tile must hold whole key-grid rows");
};

__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

template <int D, int BN, int KW, int MASK, int NS>
__global__ void __launch_bounds__(kThreads, 1) flash_fwd_tc(const __grid_constant__ TcArgs args) {
  constexpr bool kMaskTma = (MASK == TC_FLOAT_TMA || MASK == TC_BOOL_TMA);
  constexpr int kMaskElem = MASK == TC_FLOAT_TMA ? 2 : (MASK == TC_BOOL_TMA ? 1 : 0);
  static_assert(!kMaskTma || (BN == 64 && KW == 0), "TMA mask tiles: 64 keys per row");
  using L = Layout<D, BN, KW, NS, kMaskElem>;
  // head_dim 64 leaves 128 TMEM columns free: P_A [384,448), P_B [448,512) get
  // their own columns, so S_t(j+1) = Q_t.K_{j+1}^T can be issued as soon as
  // softmax t has read S_t(j), before P_t(j) exists.  At head_dim 128, P_t
  // overwrites S_t and the next Q.K^T waits for P_t.V.
  constexpr bool kPSep = (D == 64);
  // head_dim 128 with 64-key tiles: each query tile gets two 64-column S
  // buffers at [128t, 128t+64) and [128t+64, 128t+128) (O_t at 256+128t), and
  // P_t(j) is written over the first half of the S buffer it was read from.
  // S_t(j+2) goes into that buffer right after O_t += P_t(j).V_j (in issue
  // order), so the next score tile is always computed one tile ahead.
  constexpr bool kSDB = (D == 128 && BN == 64);
  constexpr bool kRwInSmem = KW >= 32;  // large key-grid width: rel_w re-read per tile
  constexpr int kRwSwz = KW >= 64 ? 15 : 7;  // float4-index XOR swizzle of those rows (conflict-free)
  extern __shared__ uint8_t smem_raw[];
  // offset from smem_raw (not a cast through an integer) so that the
  // compiler keeps the shared address space and emits shared loads
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem + L::oQ;
  uint8_t* sK = smem + L::oK;
  uint8_t* sV = smem + L::oV;
  float* sRel = reinterpret_cast<float*>(smem + L::oRel);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::oBar);
  uint64_t* k_full = bars;               // [NS]  TMA -> MMA
  uint64_t* v_full = bars + NS;          // [NS]
  uint64_t* k_empty = bars + 2 * NS;     // [NS]  MMA commit after the last Q.K^T reading K -> TMA
  uint64_t* v_empty = bars + 3 * NS;     // [NS]  MMA commit after the last P.V reading V -> TMA
  uint64_t* q_full = bars + 4 * NS;      // Q tiles (and rel tables) landed
  uint64_t* s_full = q_full + 1;         // [2]   MMA commit -> softmax t
  uint64_t* p_full = q_full + 3;         // [2]   softmax t (128 arrivals) -> MMA
  uint64_t* o_done = q_full + 5;         // [2]   final MMA commit -> softmax t epilogue
  uint64_t* rel_mma = q_full + 7;        // rel projections in TMEM (MMA commit)
  uint64_t* rel_read = q_full + 8;       // projections read by all 256 softmax threads
  uint64_t* fin = q_full + 9;            // last commit before TMEM release
  uint64_t* s_free = q_full + 10;        // [2]   softmax t read S_t (128 arrivals) -> MMA   (kPSep)
  uint64_t* o_ready = q_full + 12;       // [2]   MMA commit after each O_t += P_t V         (kPSep)
  // kSDB: O_t += P_t(j).V_j commits o_ready[t] for even j and o_odd[t] for odd
  // j, so that each barrier is at most one phase from any wait on it
  uint64_t* o_odd = q_full + 14;         // [2]
  // kSDB: likewise S_t(j) completes s_full[t] / s_odd[t] and P_t(j) arrives on
  // p_full[t] / p_odd[t] by the parity of j -- with two S buffers either side
  // can run a tile ahead, and a single barrier could then be two phases ahead
  // of its waiter
  uint64_t* s_odd = q_full + 16;         // [2]
  uint64_t* p_odd = q_full + 18;         // [2]   (128 arrivals)
  // kMaskTma: mask tile of query tile t, stage s at [2 t + s]: TMA -> softmax t,
  // and softmax t (128 arrivals) -> producer
  uint64_t* m_full = q_full + 20;        // [4]
  uint64_t* m_empty = q_full + 24;       // [4]
  uint8_t* sMask = smem + L::oMask;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + L::kBars);
  int* abort_flag = reinterpret_cast<int*>(tslot + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  // Launched behind another grid (programmatic serialization), this CTA may
  // start while that grid runs: everything before grid_dep_wait() touches
  // only kernel parameters, shared memory and TMEM.  The next grid may be
  // scheduled once every CTA of this one has started; its CTAs take SMs as
  // this grid's leave and wait for its completion there.
  grid_dep_launch();
  int unit, sidx = 0, nsplit = 1;  // sidx: which part of the unit's key range this CTA takes
  if ((int)blockIdx.x < args.n_full) {
    unit = blockIdx.x;
  } else {
    const int i = blockIdx.x - args.n_full;
    nsplit = args.n_split;
    const int pu = (int)fdiv((uint32_t)i, args.fd_split);
    unit = args.n_full + pu;
    sidx = i - pu * nsplit;
  }
  // unit = (b * Hq + h) * nqblk + qraw, or (b * nqblk + qraw) * Hq + h head-fastest
  int qraw, h, b;
  if (args.head_fast) {
    const int u1 = (int)fdiv((uint32_t)unit, args.fd_hq);
    h = unit - u1 * args.Hq;
    b = (int)fdiv((uint32_t)u1, args.fd_nqblk);
    qraw = u1 - b * args.nqblk;
  } else {
    const int u1 = (int)fdiv((uint32_t)unit, args.fd_nqblk);
    qraw = unit - u1 * args.nqblk;
    b = (int)fdiv((uint32_t)u1, args.fd_hq);
    h = u1 - b * args.Hq;
  }
  const int qblk = args.reverse_q ? args.nqblk - 1 - qraw : qraw;
  const int hk = (int)fdiv((uint32_t)h, args.fd_group);
  const int q0 = qblk * 2 * kRowsPerTile;

  // Key-tile range of the query block (causal / sliding skip whole tiles) ...
  int jb = 0, je = (args.Tkv + BN - 1) / BN;
  if (MASK == TC_RANGE) {
    const long long first = q0;
    const long long last = (long long)min(q0 + 2 * kRowsPerTile, args.Tq) - 1;
    long long lo = 0, hi = args.Tkv;
    if (last + args.offset + 1 < hi) hi = last + args.offset + 1;
    if (args.mask_kind == SDPA_MASK_SLIDING) lo = max(0LL, first + args.offset - args.window + 1);
    if (hi <= lo) {
      jb = je = 0;
    } else {
      jb = (int)(lo / BN);
      je = (int)((hi + BN - 1) / BN);
    }
  }
  // ... and this CTA's share of it
  const int j_begin = nsplit == 1 ? jb : jb + (int)fdiv((uint32_t)((je - jb) * sidx), args.fd_split);
  const int j_end = nsplit == 1 ? je : jb + (int)fdiv((uint32_t)((je - jb) * (sidx + 1)), args.fd_split);
  const int n_tiles = j_end - j_begin;
  // debug builds: the unit and its share of key tiles lie inside the problem
  // (uniform over the CTA, so the whole CTA leaves before any barrier)
  if (!dcheck(args.err, unit >= 0 && (long long)unit < (long long)args.B * args.Hq * args.nqblk && sidx < nsplit &&
                            j_begin >= 0 && j_begin <= j_end && (long long)j_end * BN < (long long)args.Tkv + BN))
    return;

  if (tid == 0) {
    *abort_flag = 0;
    for (int i = 0; i < L::kBars; ++i) mbar_init(&bars[i], 1);
    mbar_init(&p_full[0], kRowsPerTile);
    mbar_init(&p_full[1], kRowsPerTile);
    mbar_init(rel_read, 2 * kRowsPerTile);
    mbar_init(&s_free[0], kRowsPerTile);
    mbar_init(&s_free[1], kRowsPerTile);
    mbar_init(&p_odd[0], kRowsPerTile);
    mbar_init(&p_odd[1], kRowsPerTile);
    if constexpr (kMaskTma)
      for (int i = 0; i < 4; ++i) mbar_init(&m_empty[i], kRowsPerTile);
    fence_mbar_init();
    grid_dep_wait();
    if (n_tiles > 0) {
      // Q (and the rel tables) and the first K tile go out before the TMEM
      // allocation and the CTA barrier, so their latency overlaps the setup
      tma_prefetch_desc(&args.tq);
      tma_prefetch_desc(&args.tk);
      uint32_t qbytes = 2 * L::kQBytes;
      if (KW > 0) qbytes += 2 * args.rel_n * 128;
      mbar_expect_tx(q_full, qbytes);
      for (int t = 0; t < 2; ++t)
        for (int p = 0; p < L::kPanels; ++p)
          tma_load_4d(sQ + t * L::kQBytes + p * kRowsPerTile * 128, &args.tq, q_full, p * 64,
                      q0 + t * kRowsPerTile, h, b);
      if (KW > 0) {
        // the rel tables borrow the last stage's K/V buffers until the projections are done
        tma_load_3d(sK + (NS - 1) * L::kKVBytes, &args.trh, q_full, 0, 0, 0);
        tma_load_3d(sV + (NS - 1) * L::kKVBytes, &args.trw, q_full, 0, 0, 0);
      }
      mbar_expect_tx(&k_full[0], L::kKVBytes);
      for (int p = 0; p < L::kPanels; ++p)
        tma_load_4d(sK + p * BN * 128, &args.tk, &k_full[0], p * 64, j_begin * BN, hk, b);
    }
  }
  if (warp == 9) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  grid_dep_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  volatile int* abort_v = abort_flag;
  constexpr bool kWarpIssue = true;
  auto mma_ss_x = [](uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    if constexpr (kWarpIssue) mma_ss_w(d, a, b, id, acc); else mma_ss(d, a, b, id, acc);
  };
  auto mma_ts_x = [](uint32_t d, uint32_t a, uint64_t b, uint32_t id, uint32_t acc) {
    if constexpr (kWarpIssue) mma_ts_w(d, a, b, id, acc); else mma_ts(d, a, b, id, acc);
  };
  auto mma_commit_x = [](uint64_t* bar) {
    if constexpr (kWarpIssue) mma_commit_w(bar); else mma_commit(bar);
  };
  auto wait_x = [](bool v) {
    if constexpr (kWarpIssue) return __all_sync(0xffffffffu, v); else return v;
  };

  // Register split: the producer/MMA warpgroup gives registers to the two
  // softmax warpgroups (3 x 128 x 168 at launch = 2 x 128 x 232 + 128 x 40).
  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kRegsOther));
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&args.tv);
      // K runs one tile ahead of V: a K stage frees as soon as both Q.K^T
      // products that read it are done, a V stage only after both P.V.
      // Q, the rel tables and K tile 0 were issued during setup.
      bool ok = true;
      int k_issued = 1, v_issued = 0;
      auto load_k = [&](int jj) {
        const int s = jj % NS, use = jj / NS;
        if (use > 0) ok = mbar_wait(&k_empty[s], (use - 1) & 1, abort_v, args.err);
        if (ok && KW > 0 && jj == NS - 1) ok = mbar_wait(rel_mma, 0, abort_v, args.err);
        if (!ok) return;
        const int key0 = (j_begin + jj) * BN;
        mbar_expect_tx(&k_full[s], L::kKVBytes);
        for (int p = 0; p < L::kPanels; ++p)
          tma_load_4d(sK + s * L::kKVBytes + p * BN * 128, &args.tk, &k_full[s], p * 64, key0, hk, b);
        k_issued = jj + 1;
      };
      auto load_v = [&](int jj) {
        const int s = jj % NS, use = jj / NS;
        if (use > 0) ok = mbar_wait(&v_empty[s], (use - 1) & 1, abort_v, args.err);
        if (ok && KW > 0 && jj == NS - 1) ok = mbar_wait(rel_mma, 0, abort_v, args.err);
        if (!ok) return;
        const int key0 = (j_begin + jj) * BN;
        mbar_expect_tx(&v_full[s], L::kKVBytes);
        for (int p = 0; p < L::kPanels; ++p)
          tma_load_4d(sV + s * L::kKVBytes + p * BN * 128, &args.tv, &v_full[s], p * 64, key0, hk, b);
        v_issued = jj + 1;
      };
      // kMaskTma: both query tiles' mask tiles of key tile jj, in stage jj & 1
      int m_issued = 0;
      auto load_m = [&](int jj) {
        if constexpr (kMaskTma) {
          // both query tiles' stages free first, then both loads: a wait that
          // gives up leaves no load of this key tile in flight
          const int s = jj & 1, use = jj >> 1;
          for (int t = 0; t < 2 && ok && use > 0; ++t)
            ok = mbar_wait(&m_empty[2 * t + s], (use - 1) & 1, abort_v, args.err);
          if (!ok) return;
          for (int t = 0; t < 2; ++t) {
            mbar_expect_tx(&m_full[2 * t + s], L::kMaskBytes);
            tma_load_4d(sMask + (2 * t + s) * L::kMaskBytes, &args.tm, &m_full[2 * t + s], (j_begin + jj) * BN,
                        q0 + t * kRowsPerTile, args.msh ? h : 0, args.msb ? b : 0);
          }
          m_issued = jj + 1;
        }
      };
      if constexpr (kMaskTma) tma_prefetch_desc(&args.tm);
      load_m(0);
      constexpr int kAhead = kSDB ? 2 : 1;  // K tiles loaded ahead of V (the MMA issues S two tiles ahead in kSDB)
      for (int jj = 1; jj < n_tiles && ok; ++jj) {
        load_k(jj);
        if (ok && jj >= kAhead) load_v(jj - kAhead);
        if (ok) load_m(jj);
      }
      for (int jv = max(0, n_tiles - kAhead); jv < n_tiles && ok; ++jv) load_v(jv);
      if (!ok) {
        // abandoned: let the copies already in flight land before the CTA exits
        if constexpr (kMaskTma)
          for (int jj = max(0, m_issued - 2); jj < m_issued; ++jj)
            for (int t = 0; t < 2; ++t) mbar_wait(&m_full[2 * t + (jj & 1)], (jj >> 1) & 1, nullptr, args.err);
        mbar_wait(q_full, 0, nullptr, args.err);
        for (int jj = max(0, k_issued - NS); jj < k_issued; ++jj)
          mbar_wait(&k_full[jj % NS], (jj / NS) & 1, nullptr, args.err);
        for (int jj = max(0, v_issued - NS); jj < v_issued; ++jj)
          mbar_wait(&v_full[jj % NS], (jj / NS) & 1, nullptr, args.err);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (every wait is warp-uniform) and one elected
    // lane issues each instruction: measured faster than lane 0 running it
    // alone (SAM global attention, head_dim 64: 100.4 against 110.8 us).
    if ((kWarpIssue || lane == 0) && n_tiles > 0) {
      constexpr uint32_t id_qk = idesc_bf16_f32(128, BN, false, false);
      constexpr uint32_t id_pv = idesc_bf16_f32(128, D, false, true);
      // Descriptors are built once; a byte offset inside shared memory is added
      // to the start-address field (address >> 4, no carry out of 14 bits).
      const uint64_t dq = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dk = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dv = sdesc_sw128(smem_u32(sV), BN * 128, 1024);
      bool ok = wait_x(mbar_wait(q_full, 0, abort_v, args.err));
      auto qk = [&](int t, int s, int buf = 0) {
        const uint64_t a0 = dq + (uint64_t)((t * L::kQBytes) >> 4);
        const uint64_t b0 = dk + (uint64_t)((s * L::kKVBytes) >> 4);
        const uint32_t d_tm = tbase + t * 128 + buf * 64;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ao = ((kk >> 2) * (kRowsPerTile * 128) + (kk & 3) * 32) >> 4;
          const uint32_t bo = ((kk >> 2) * (BN * 128) + (kk & 3) * 32) >> 4;
          mma_ss_x(d_tm, a0 + ao, b0 + bo, id_qk, kk > 0);
        }
      };
      auto pv = [&](int t, int s, bool first, int buf = 0) {
        const uint64_t b0 = dv + (uint64_t)((s * L::kKVBytes) >> 4);
        const uint32_t d_tm = tbase + 256 + t * D;
        const uint32_t a_tm = kPSep ? tbase + 384 + t * 64 : tbase + t * 128 + buf * 64;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ts_x(d_tm, a_tm + kk * 8, b0 + (uint64_t)((kk * 16 * 128) >> 4), id_pv, (!first) || kk > 0);
      };
      if (ok && KW > 0) {
        // rel projections: Ph_t -> cols [256t, 256t+rel_n), Pw_t -> [256t+128, 256t+128+rel_n)
        const uint32_t id_rel = idesc_bf16_f32(128, args.rel_n, false, false);
        const uint64_t drh = dk + (uint64_t)(((NS - 1) * L::kKVBytes) >> 4);
        const uint64_t drw = sdesc_sw128(smem_u32(sV + (NS - 1) * L::kKVBytes), 16, 1024);
        tc_fence_after();
        for (int t = 0; t < 2; ++t)
          for (int w = 0; w < 2; ++w)
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_ss_x(tbase + t * 256 + w * 128, dq + (uint64_t)((t * L::kQBytes + kk * 32) >> 4),
                     (w == 0 ? drh : drw) + (uint64_t)((kk * 32) >> 4), id_rel, kk > 0);
        mma_commit_x(rel_mma);
        ok = wait_x(mbar_wait(rel_read, 0, abort_v, args.err));
      }
      // prologue: S_A(0), S_B(0)
      if (ok) ok = wait_x(mbar_wait(&k_full[0], 0, abort_v, args.err));
      if (ok) {
        tc_fence_after();
        qk(0, 0);
        mma_commit_x(&s_full[0]);
        qk(1, 0);
        mma_commit_x(&s_full[1]);
        mma_commit_x(&k_empty[0]);
      }
      if (kSDB && ok && n_tiles > 1) {
        ok = wait_x(mbar_wait(&k_full[1], 0, abort_v, args.err));
        if (ok) {
          tc_fence_after();
          qk(0, 1, 1);
          mma_commit_x(&s_odd[0]);
          qk(1, 1, 1);
          mma_commit_x(&s_odd[1]);
          mma_commit_x(&k_empty[1]);
        }
      }
      if constexpr (kSDB) {
        // O_t += P_t(j).V_j, then S_t(j+2) into the buffer P_t(j) was read from
        for (int jj = 0; jj < n_tiles && ok; ++jj) {
          const int s = jj % NS, buf = jj & 1;
          const bool more = jj + 2 < n_tiles;
          const int s2 = (jj + 2) % NS;
          ok = wait_x(mbar_wait(&v_full[s], (jj / NS) & 1, abort_v, args.err));
          if (ok) ok = wait_x(mbar_wait(buf ? &p_odd[0] : &p_full[0], (jj >> 1) & 1, abort_v, args.err));
          if (!ok) break;
          tc_fence_after();
          pv(0, s, jj == 0, buf);
          mma_commit_x(jj & 1 ? &o_odd[0] : &o_ready[0]);
          if (more) {
            ok = wait_x(mbar_wait(&k_full[s2], ((jj + 2) / NS) & 1, abort_v, args.err));
            if (!ok) break;
            tc_fence_after();
            qk(0, s2, buf);
            mma_commit_x(buf ? &s_odd[0] : &s_full[0]);
          }
          ok = wait_x(mbar_wait(buf ? &p_odd[1] : &p_full[1], (jj >> 1) & 1, abort_v, args.err));
          if (!ok) break;
          tc_fence_after();
          pv(1, s, jj == 0, buf);
          mma_commit_x(jj & 1 ? &o_odd[1] : &o_ready[1]);
          mma_commit_x(&v_empty[s]);
          if (more) {
            qk(1, s2, buf);
            mma_commit_x(buf ? &s_odd[1] : &s_full[1]);
            mma_commit_x(&k_empty[s2]);
          }
        }
      } else if constexpr (kPSep) {
        // A and B alternate: S_A(j+1), O_A += P_A(j).V_j, S_B(j+1), O_B += P_B(j).V_j
        for (int jj = 0; jj < n_tiles && ok; ++jj) {
          const int s = jj % NS;
          const bool more = jj + 1 < n_tiles;
          const int s1 = (jj + 1) % NS;
          if (more) {
            ok = wait_x(mbar_wait(&k_full[s1], ((jj + 1) / NS) & 1, abort_v, args.err));
            if (ok) ok = wait_x(mbar_wait(&s_free[0], jj & 1, abort_v, args.err));
            if (!ok) break;
            tc_fence_after();
            qk(0, s1);
            mma_commit_x(&s_full[0]);
          }
          ok = wait_x(mbar_wait(&v_full[s], (jj / NS) & 1, abort_v, args.err));
          if (ok) ok = wait_x(mbar_wait(&p_full[0], jj & 1, abort_v, args.err));
          if (!ok) break;
          tc_fence_after();
          pv(0, s, jj == 0);
          mma_commit_x(&o_ready[0]);
          if (more) {
            ok = wait_x(mbar_wait(&s_free[1], jj & 1, abort_v, args.err));
            if (!ok) break;
            tc_fence_after();
            qk(1, s1);
            mma_commit_x(&s_full[1]);
            mma_commit_x(&k_empty[s1]);
          }
          ok = wait_x(mbar_wait(&p_full[1], jj & 1, abort_v, args.err));
          if (!ok) break;
          tc_fence_after();
          pv(1, s, jj == 0);
          mma_commit_x(&o_ready[1]);
          mma_commit_x(&v_empty[s]);
        }
      } else {
        for (int jj = 0; jj < n_tiles && ok; ++jj) {
          const int s = jj % NS;
          ok = wait_x(mbar_wait(&v_full[s], (jj / NS) & 1, abort_v, args.err));
          if (!ok) break;
          // tile A: O_A += P_A V_j, then S_A(j+1)
          ok = wait_x(mbar_wait(&p_full[0], jj & 1, abort_v, args.err));
          if (!ok) break;
          tc_fence_after();
          pv(0, s, jj == 0);
          const bool more = jj + 1 < n_tiles;
          const int s1 = (jj + 1) % NS;
          if (more) {
            ok = wait_x(mbar_wait(&k_full[s1], ((jj + 1) / NS) & 1, abort_v, args.err));
            if (!ok) break;
            tc_fence_after();
            qk(0, s1);
            mma_commit_x(&s_full[0]);
          }
          // tile B: O_B += P_B V_j, release V_j, then S_B(j+1) and release K_{j+1}
          ok = wait_x(mbar_wait(&p_full[1], jj & 1, abort_v, args.err));
          if (!ok) break;
          tc_fence_after();
          pv(1, s, jj == 0);
          mma_commit_x(&v_empty[s]);
          if (more) {
            qk(1, s1);
            mma_commit_x(&s_full[1]);
            mma_commit_x(&k_empty[s1]);
          }
        }
      }
      mma_commit_x(&o_done[0]);
      mma_commit_x(&o_done[1]);
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kRegsSoftmax));
    // ------------------------------------------------------------ softmax of tile t
    const int t = warp >> 2;
    const int lr = (warp & 3) * 32 + lane;   // row within the tile = TMEM lane
    const int row = t * kRowsPerTile + lr;   // row within the CTA
    const long long qi = (long long)q0 + row;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_base = tbase + lane_off + t * 128;
    const uint32_t o_addr = tbase + lane_off + 256 + t * D;
    const uint32_t p_fixed = tbase + lane_off + 384 + t * 64;  // kPSep
    bool ok = true;
    float* relh_s = sRel;                   // [kRelHMax][256]
    float* relw_s = sRel + kRelHMax * 256;  // [KW][256], or [256][KW] (swizzled) when read as float4 per tile

    if constexpr (KW > 0) if (n_tiles > 0) {
      // scatter this row's rel_h / rel_w (log2 e prescaled) into shared memory
      ok = __all_sync(0xffffffffu, mbar_wait(rel_mma, 0, abort_v, args.err));
      tc_fence_after();
      const int qw_n = args.qw_n, kh_n = args.kh_n;
      const int qh = (int)fdiv((uint32_t)qi, args.fd_qw), qw = (int)qi - qh * qw_n;
      if (ok) {
        // rolled over w and the chunks: this code runs once per CTA, from a
        // cold instruction cache
#pragma unroll 1
        for (int w = 0; w < 2; ++w) {
          // key-grid coordinate k of this row is reached through table row
          // (= projection column) base - k, 0 <= k < nk
          const int base_idx = w == 0 ? qh + kh_n - 1 : qw + KW - 1;
          const unsigned nk = w == 0 ? kh_n : KW;
          // the columns any row of this warp takes (when a warp shares one
          // query-grid row and spans 32 grid columns, at most three of the four
          // 32-column chunks)
          const int c_lo = __reduce_min_sync(0xffffffffu, base_idx) - (int)nk + 1;
          const int c_hi = __reduce_max_sync(0xffffffffu, base_idx);
          float* dst_h = w == 0 ? relh_s : relw_s;
          const bool swz = w == 1 && kRwInSmem;
#pragma unroll 1
          for (int c0 = 0; c0 < 128; c0 += 32) {
            if (c0 < args.rel_n && c0 + 31 >= c_lo && c0 <= c_hi) {
              uint32_t r[32];
              tmem_ld32(tbase + lane_off + t * 256 + w * 128 + c0, r);
              tmem_wait_ld();
              const int kb = base_idx - c0;
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int k = kb - i;
                if ((unsigned)k < nk && dcheck_idx(args.err, k, w == 0 ? kRelHMax : KW)) {
                  const float val = __uint_as_float(r[i]) * kLog2e;
                  if (swz)
                    // this row's slice, float4 groups XOR-swizzled by row (float4
                    // group g at g ^ (row & kRwSwz), i.e. element k at
                    // k ^ ((row & kRwSwz) << 2)): the loop reads it as float4
                    // without bank conflicts, and so does this scatter when the
                    // query and key grids have equal width
                    relw_s[row * KW + (k ^ ((row & kRwSwz) << 2))] = val;
                  else
                    // [k][256]: consecutive rows hit consecutive banks whatever k is
                    dst_h[k * 256 + row] = val;
                }
              }
            }
          }
        }
      }
      // every thread reads back only what it wrote itself: no CTA barrier is
      // needed before the loop
      tc_fence_before();
      mbar_arrive(rel_read);
    }

    // per-row visible key range (causal / sliding)
    long long lo_i = 0, hi_i = args.Tkv;
    if constexpr (MASK == TC_RANGE) {
      if (qi + args.offset + 1 < hi_i) hi_i = qi + args.offset + 1;
      if (args.mask_kind == SDPA_MASK_SLIDING) lo_i = max(0LL, qi + args.offset - args.window + 1);
    }
    const bool row_valid = qi < args.Tq;
    const long long mrow = (long long)b * args.msb + (long long)h * args.msh + qi * args.msq;

    // rel_w of this row: in registers for the whole loop when small, else
    // re-read per tile as float4 from this row's shared-memory slice (log2 units)
    float rw[(KW > 0 && !kRwInSmem) ? KW : 2];
    if constexpr (KW > 0 && !kRwInSmem) {
#pragma unroll
      for (int c = 0; c < KW; ++c) rw[c] = relw_s[c * 256 + row];
    }
    const float4* rw4 = reinterpret_cast<const float4*>(relw_s + row * (KW > 0 ? KW : 1));
    constexpr int NG = KW > 0 ? BN / KW : 1;  // key-grid rows per key tile (1 without rel-pos)
    constexpr int GW = BN / NG;                // keys per group
    static_assert(GW % 2 == 0, "groups hold whole pairs");
    const uint64_t sl2 = f2(args.scale_log2, args.scale_log2);

    float m_run = -INFINITY, l_run = 0.f;
    for (int jj = 0; jj < n_tiles && ok; ++jj) {
      const int j0 = (j_begin + jj) * BN;
      if constexpr (kSDB)
        ok = __all_sync(0xffffffffu, mbar_wait(jj & 1 ? &s_odd[t] : &s_full[t], (jj >> 1) & 1, abort_v, args.err));
      else
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[t], jj & 1, abort_v, args.err));
      if (!ok) break;
      tc_fence_after();
      // this tile's S columns (and, unless P has its own, where P goes)
      const uint32_t s_addr = s_base + (kSDB ? (jj & 1) * 64 : 0);
      const uint32_t p_addr = kPSep ? p_fixed : s_addr;
      uint32_t sr[BN];
#pragma unroll
      for (int c0 = 0; c0 < BN; c0 += 32) {
        if (c0 + 32 <= BN)
          tmem_ld32p(s_addr + c0, sr + c0);
        else
          tmem_ld16p(s_addr + c0, sr + c0);
      }
      tmem_wait_ld();
      if constexpr (kPSep) {
        tc_fence_before();
        mbar_arrive(&s_free[t]);
      }

      // x = s*scale (+ rel_w) in log2 units, two columns per instruction; rel_h
      // is constant over a key-grid row, so it is kept per group (goff) and
      // folded into the max and the exponent.
      uint64_t x2[BN / 2];
      float goff[NG];
      if constexpr (KW > 0) {
        const int kh0 = j0 / KW;
#pragma unroll
        for (int g = 0; g < NG; ++g) {
          const int khi = kh0 + g;
          goff[g] = khi < args.kh_n ? relh_s[khi * 256 + row] : 0.f;
        }
        if constexpr (kRwInSmem) {
#pragma unroll
          for (int c = 0; c < KW; c += 4) {
            const float4 w4 = rw4[(c / 4) ^ (row & kRwSwz)];
            const uint64_t wa = f2(w4.x, w4.y), wb = f2(w4.z, w4.w);
#pragma unroll
            for (int g = 0; g < NG; ++g) {
              const int e = g * KW + c;
              x2[e / 2] = f2_fma(f2u(sr[e], sr[e + 1]), sl2, wa);
              x2[e / 2 + 1] = f2_fma(f2u(sr[e + 2], sr[e + 3]), sl2, wb);
            }
          }
        } else {
#pragma unroll
          for (int g = 0; g < NG; ++g)
#pragma unroll
            for (int c = 0; c < KW; c += 2) {
              const int e = g * KW + c;
              x2[e / 2] = f2_fma(f2u(sr[e], sr[e + 1]), sl2, f2(rw[c], rw[c + 1]));
            }
        }
      } else {
        goff[0] = 0.f;
#pragma unroll
        for (int i = 0; i < BN / 2; ++i) x2[i] = f2_mul(f2u(sr[2 * i], sr[2 * i + 1]), sl2);
      }

      // masks (scalar, only on tiles that need them)
      auto set_ninf = [&](int c) {
        float lo, hi;
        f2_split(x2[c / 2], lo, hi);
        if (c & 1) hi = -INFINITY; else lo = -INFINITY;
        x2[c / 2] = f2(lo, hi);
      };
      if constexpr (MASK == TC_RANGE) {
        if (!(j0 >= lo_i && j0 + BN <= hi_i)) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (j0 + c < lo_i || j0 + c >= hi_i) set_ninf(c);
        }
      } else if constexpr (MASK == TC_FLOAT) {
        if (row_valid) {
          const __nv_bfloat16* mp = static_cast<const __nv_bfloat16*>(args.mask) + mrow + j0;
          const uint64_t l2e = f2(kLog2e, kLog2e);
          if (j0 + BN <= args.Tkv && args.mask_vec) {
#pragma unroll
            for (int c = 0; c < BN; c += 8) {
              const uint4 raw = __ldg(reinterpret_cast<const uint4*>(mp + c));
              const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
              for (int u = 0; u < 4; ++u)  // bf16 pair -> fp32 pair by moving each half to the top 16 bits
                x2[c / 2 + u] = f2_fma(f2u(wv[u] << 16, wv[u] & 0xFFFF0000u), l2e, x2[c / 2 + u]);
            }
          } else {
#pragma unroll
            for (int c = 0; c < BN; c += 2) {
              const float m0 = j0 + c < args.Tkv ? __bfloat162float(mp[c]) : 0.f;
              const float m1 = j0 + c + 1 < args.Tkv ? __bfloat162float(mp[c + 1]) : 0.f;
              x2[c / 2] = f2_fma(f2(m0, m1), l2e, x2[c / 2]);
            }
          }
        }
      } else if constexpr (kMaskTma) {
        // this row of the tile's mask from shared memory: 128 bytes of bf16 in
        // the 128-byte swizzle (16-byte piece c at c ^ (row & 7)), or 64 bytes
        // of bool in the 64-byte swizzle (piece c at c ^ ((row >> 1) & 3)).
        // Rows past Tq and keys past Tkv were filled with zeros: a zero bool
        // hides a key, which is right for those keys (and their rows are
        // never stored); float keys past Tkv are set to -inf below.
        const int ms = 2 * t + (jj & 1);
        ok = __all_sync(0xffffffffu, mbar_wait(&m_full[ms], (jj >> 1) & 1, abort_v, args.err));
        if (!ok) break;
        const int rt = row & (kRowsPerTile - 1);
        const uint8_t* mrow_s = sMask + ms * L::kMaskBytes + rt * (BN * kMaskElem);
        if constexpr (MASK == TC_FLOAT_TMA) {
          const uint64_t l2e = f2(kLog2e, kLog2e);
#pragma unroll
          for (int c = 0; c < BN; c += 8) {
            const uint4 raw = *reinterpret_cast<const uint4*>(mrow_s + (((c >> 3) ^ (rt & 7)) << 4));
            const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int u = 0; u < 4; ++u)  // bf16 pair -> fp32 pair by moving each half to the top 16 bits
              x2[c / 2 + u] = f2_fma(f2u(wv[u] << 16, wv[u] & 0xFFFF0000u), l2e, x2[c / 2 + u]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < BN; c += 16) {
            const uint4 raw = *reinterpret_cast<const uint4*>(mrow_s + (((c >> 4) ^ ((rt >> 1) & 3)) << 4));
            const uint8_t* e = reinterpret_cast<const uint8_t*>(&raw);
#pragma unroll
            for (int u = 0; u < 16; ++u)
              if (e[u] == 0) set_ninf(c + u);
          }
        }
        mbar_arrive(&m_empty[ms]);
      } else if constexpr (MASK == TC_BOOL) {
        if (row_valid) {
          const uint8_t* mp = static_cast<const uint8_t*>(args.mask) + mrow + j0;
          if (j0 + BN <= args.Tkv && args.mask_vec) {
#pragma unroll
            for (int c = 0; c < BN; c += 16) {
              const uint4 raw = __ldg(reinterpret_cast<const uint4*>(mp + c));
              const uint8_t* e = reinterpret_cast<const uint8_t*>(&raw);
#pragma unroll
              for (int u = 0; u < 16; ++u)
                if (e[u] == 0) set_ninf(c + u);
            }
          } else {
#pragma unroll
            for (int c = 0; c < BN; ++c)
              if (j0 + c < args.Tkv && mp[c] == 0) set_ninf(c);
          }
        }
      }
      if (j0 + BN > args.Tkv) {
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (j0 + c >= args.Tkv) set_ninf(c);
      }

      const float mx = tile::row_max<NG, GW>(x2, goff);
      const float m_new = fmaxf(m_run, mx);
      const bool need = m_new > m_run + kRescaleThreshold;  // false while both are -inf
      float alpha = 1.f;
      if (need) {
        alpha = ex2_approx(m_run - m_new);  // 0 when m_run == -inf
        l_run *= alpha;
        m_run = m_new;
      }
      // p = 2^(x + goff - m), packed to bf16 pairs in registers first, so that
      // the wait for the previous P.V below comes after the exponentials.
      const float m_use = m_run == -INFINITY ? 0.f : m_run;
      uint32_t pk[BN / 2];
      l_run += tile::exp_pack<BN, GW>(x2, goff, m_use, pk);
      if constexpr (kPSep) {
        // O_t += P_t(j-1).V_{j-1} must be complete before O_t is rescaled or P_t is overwritten
        if (jj > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(&o_ready[t], (jj - 1) & 1, abort_v, args.err));
          if (!ok) break;
          tc_fence_after();
        }
      }
      const bool rescale = jj > 0 && __any_sync(0xffffffffu, need);
      if constexpr (kSDB) {
        // P_t(j) overwrites a buffer whose last reader, P_t(j-2).V, completed
        // before S_t(j) (same commit); only a rescale of O_t waits for
        // O_t += P_t(j-1).V, on the barrier of its parity: P_t(j-3).V is done
        // and P_t(j+1).V cannot be, so that barrier is within one phase
        if (rescale) {
          const int x = jj - 1;
          ok = __all_sync(0xffffffffu, mbar_wait(x & 1 ? &o_odd[t] : &o_ready[t], (x >> 1) & 1, abort_v, args.err));
          if (!ok) break;
          tc_fence_after();
        }
      }
      if (rescale) tile::rescale_o<D>(o_addr, alpha);  // O_t row *= alpha
      tile::store_p<BN>(p_addr, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(kSDB && (jj & 1) ? &p_odd[t] : &p_full[t]);
    }

    // epilogue: O / l -> bf16, rows past Tq are not stored
    const long long zq = (long long)b * args.Hq + h;
    __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(args.out) + (long long)b * args.sob + (long long)h * args.soh + qi * args.sot;
    if (n_tiles > 0 && ok) {
      if constexpr (kSDB) {
        // the last two P.V may both be in flight, one on each parity's barrier
        for (int x = max(0, n_tiles - 2); x < n_tiles && ok; ++x)
          ok = __all_sync(0xffffffffu, mbar_wait(x & 1 ? &o_odd[t] : &o_ready[t], (x >> 1) & 1, abort_v, args.err));
      } else if constexpr (kPSep) {
        ok = __all_sync(0xffffffffu, mbar_wait(&o_ready[t], (n_tiles - 1) & 1, abort_v, args.err));
      }
      else
        ok = __all_sync(0xffffffffu, mbar_wait(&o_done[t], 0, abort_v, args.err));
      tc_fence_after();
    }
    if (nsplit == 1) {
      if (n_tiles == 0) {
        if (row_valid) {
#pragma unroll
          for (int c = 0; c < D; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
          if (args.lse) args.lse[zq * args.Tq + qi] = -INFINITY;
        }
      } else if (ok) {
        // O / l as bf16 rows staged in this query tile's Q buffer (dead: the
        // tile's last Q.K^T has completed), in the Q load's own 128-byte
        // swizzle, then one TMA store per 64-column panel of the warp's 32
        // rows (rows past Tq are not written)
        uint8_t* stage = sQ + t * L::kQBytes + (warp & 3) * 32 * 128;
        tile::stage_o_row_sw128<D>(o_addr, l_run > 0.f ? 1.f / l_run : 0.f, stage + lane * 128, lane,
                                   kRowsPerTile * 128);
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) {
          const int r0 = q0 + t * kRowsPerTile + (warp & 3) * 32;
          if (r0 < args.Tq) {
            for (int pnl = 0; pnl < L::kPanels; ++pnl)
              tma_store_4d(&args.to, stage + pnl * kRowsPerTile * 128, pnl * 64, r0, h, b);
            bulk_commit();
            bulk_wait_read_all();  // shared memory must stay until the stores have read it
          }
        }
        if (row_valid && args.lse)
          args.lse[zq * args.Tq + qi] = l_run > 0.f ? m_run * kLn2 + logf(l_run) : -INFINITY;
      }
    } else {
      // Split key range: publish this part (O unnormalised, running max m in
      // log2 units, sum l); the last CTA of the unit to arrive combines the
      // parts, O = sum_k 2^(m_k - M) O_k / sum_k 2^(m_k - M) l_k with M = max_k m_k.
      const long long part0 = (long long)(unit - args.n_full) * nsplit;
      const bool live = n_tiles > 0 && ok;  // warp-uniform: the TMEM loads are warp-collective
      const bool have = live && l_run > 0.f;
      // partial O as [part][D/4][256 rows] float4: one store instruction of a
      // warp writes 512 contiguous bytes
      float4* wso = reinterpret_cast<float4*>(args.ws_o) + (part0 + sidx) * (D / 4) * 256 + row;
      const bool ws_ok = dcheck_idx(args.err, part0 + sidx, (long long)gridDim.x - args.n_full);
      if (live) {
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(o_addr + c0, r);
          tmem_wait_ld();
          if (have && ws_ok) {
#pragma unroll
            for (int c = 0; c < 32; c += 4)
              __stcg(wso + ((c0 + c) / 4) * 256,
                     make_float4(__uint_as_float(r[c]), __uint_as_float(r[c + 1]), __uint_as_float(r[c + 2]),
                                 __uint_as_float(r[c + 3])));
          }
        }
      }
      if (ws_ok)
        __stcg(args.ws_ml + (part0 + sidx) * 256 + row, make_float2(have ? m_run : -INFINITY, have ? l_run : 0.f));
      // The barrier orders every thread's stores before thread 0's gpu-scope
      // fence and ticket increment (fences are cumulative); the last arriver's
      // fence after its increment acquires the other parts' stores.
      named_bar_sync(1, 2 * kRowsPerTile);
      if (tid == 0) {
        fence_acq_rel_gpu();
        const int last = atomicAdd(args.ws_cnt + (unit - args.n_full), 1) == nsplit - 1;
        if (last) fence_acq_rel_gpu();
        *reinterpret_cast<volatile int*>(abort_flag + 1) = last;
      }
      named_bar_sync(1, 2 * kRowsPerTile);
      if (*reinterpret_cast<volatile int*>(abort_flag + 1)) {
        // all (m, l) first (independent loads), then the weighted sum; this
        // CTA's own part is still in TMEM
        float2 ml[kMaxSplit];
        float M = have ? m_run : -INFINITY;
#pragma unroll
        for (int k = 0; k < kMaxSplit; ++k) {
          ml[k] = make_float2(-INFINITY, 0.f);
          if (k < nsplit && k != sidx) ml[k] = __ldcg(args.ws_ml + (part0 + k) * 256 + row);
          if (ml[k].y > 0.f) M = fmaxf(M, ml[k].x);
        }
        float acc[D];
        const float w_own = have ? ex2_approx(m_run - M) : 0.f;
        float den = have ? w_own * l_run : 0.f;
#pragma unroll
        for (int c = 0; c < D; ++c) acc[c] = 0.f;
        if (live) {
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(o_addr + c0, r);
            tmem_wait_ld();
            if (have) {
#pragma unroll
              for (int c = 0; c < 32; ++c) acc[c0 + c] = w_own * __uint_as_float(r[c]);
            }
          }
        }
        // the other parts' O rows are loaded whether or not the part saw a
        // key (a part without one may have left its slot unwritten: its rows
        // are then not added), so the loads need not wait for (m, l)
#pragma unroll
        for (int k = 0; k < kMaxSplit; ++k) {
          if (k < nsplit && k != sidx) {
            const bool add = ml[k].y > 0.f;
            const float w = add ? ex2_approx(ml[k].x - M) : 0.f;
            den = fmaf(w, ml[k].y, den);
            const float4* src = reinterpret_cast<const float4*>(args.ws_o) + (part0 + k) * (D / 4) * 256 + row;
#pragma unroll
            for (int c = 0; c < D; c += 4) {
              const float4 o4 = __ldcg(src + (c / 4) * 256);
              acc[c] = add ? fmaf(w, o4.x, acc[c]) : acc[c];
              acc[c + 1] = add ? fmaf(w, o4.y, acc[c + 1]) : acc[c + 1];
              acc[c + 2] = add ? fmaf(w, o4.z, acc[c + 2]) : acc[c + 2];
              acc[c + 3] = add ? fmaf(w, o4.w, acc[c + 3]) : acc[c + 3];
            }
          }
        }
        const float inv = den > 0.f ? 1.f / den : 0.f;
        if (row_valid) {
#pragma unroll
          for (int c = 0; c < D; c += 8) {
            uint4 v;
            v.x = pack_bf16x2(acc[c + 0] * inv, acc[c + 1] * inv);
            v.y = pack_bf16x2(acc[c + 2] * inv, acc[c + 3] * inv);
            v.z = pack_bf16x2(acc[c + 4] * inv, acc[c + 5] * inv);
            v.w = pack_bf16x2(acc[c + 6] * inv, acc[c + 7] * inv);
            *reinterpret_cast<uint4*>(orow + c) = v;
          }
          if (args.lse) args.lse[zq * args.Tq + qi] = den > 0.f ? M * kLn2 + logf(den) : -INFINITY;
        }
        if (tid == 0) args.ws_cnt[unit - args.n_full] = 0;  // ready for the next launch
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) {
    if (lane == 0 && n_tiles > 0) {
      // nothing this CTA issued may still be writing TMEM when it is released
      mma_commit(fin);
      mbar_wait(fin, 0, nullptr, args.err);
    }
    __syncwarp();
    tmem_dealloc(tbase, 512);
  }
}

// ---------------------------------------------------------------- host side
template <int D, int BN, int KW, int MASK, int NS>
cudaError_t launch_one(const TcArgs& a, dim3 grid, cudaStream_t stream) {
  using L = Layout<D, BN, KW, NS, MASK == TC_FLOAT_TMA ? 2 : (MASK == TC_BOOL_TMA ? 1 : 0)>;
  auto kern = flash_fwd_tc<D, BN, KW, MASK, NS>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    // setmaxnreg.inc waits for registers the CTA was launched with: refuse to
    // launch unless the split adds up against the compiled register count.
    cudaFuncAttributes fa;
    if (attr_err == cudaSuccess) attr_err = cudaFuncGetAttributes(&fa, kern);
    if (attr_err == cudaSuccess && fa.numRegs != kRegsLaunch) attr_err = cudaErrorInvalidConfiguration;
  });
  if (attr_err != cudaSuccess) return attr_err;
  // programmatic serialization: this grid's CTAs may be scheduled before the
  // previous grid in the stream completes (the kernel waits for it before it
  // touches global memory), hiding the launch gap between consecutive calls
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = L::kAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int D, int BN, int KW, int NS>
cudaError_t dispatch_mask(int mk, const TcArgs& a, dim3 grid, cudaStream_t stream) {
  switch (mk) {
    case TC_NONE: return launch_one<D, BN, KW, TC_NONE, NS>(a, grid, stream);
    case TC_RANGE: return launch_one<D, BN, KW, TC_RANGE, NS>(a, grid, stream);
    case TC_FLOAT: return launch_one<D, BN, KW, TC_FLOAT, NS>(a, grid, stream);
    case TC_BOOL: return launch_one<D, BN, KW, TC_BOOL, NS>(a, grid, stream);
  }
  return cudaErrorInvalidValue;
}


bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int tc_mask_code(const Params& p) {
  switch (p.mask_kind) {
    case SDPA_MASK_NONE: return TC_NONE;
    case SDPA_MASK_CAUSAL:
    case SDPA_MASK_SLIDING: return TC_RANGE;
    case SDPA_MASK_ADD_FLOAT: return TC_FLOAT;
    case SDPA_MASK_BOOL: return TC_BOOL;
  }
  return -1;
}

}  // namespace

// Rows of the larger rel table (Qh + Kh - 1 or Qw + Kw - 1), padded to a
// multiple of 16: the N of the projection MMAs and the TMA box height.
static int rel_rows_padded(const Params& p) {
  const int nh = p.qh_n + p.kh_n - 1, nw = p.qw_n + p.kw_n - 1;
  return ((nh > nw ? nh : nw) + 15) / 16 * 16;
}

// Whether the tensor-core kernel takes this (already validated) problem;
// SDPA_OK, SDPA_ERR_UNSUPPORTED or SDPA_ERR_MISALIGNED.
int tc_check(const Params& p, sdpa_dtype_t dtype) {
  if (dtype != SDPA_BF16) return SDPA_ERR_UNSUPPORTED;
  if (p.d != 64 && p.d != 128) return SDPA_ERR_UNSUPPORTED;
  if (p.Tkv < 1 || p.Tq < 1) return SDPA_ERR_UNSUPPORTED;
  if (p.B > 65535 || p.Hq > 65535) return SDPA_ERR_UNSUPPORTED;
  if (!al16(p.q) || !al16(p.k) || !al16(p.v) || !al16(p.out)) return SDPA_ERR_MISALIGNED;
  // TMA: byte strides multiples of 16 and below 2^40
  if (!strides_multiple_of(p, 8)) return SDPA_ERR_MISALIGNED;
  {
    const long long s[12] = {p.sqb, p.sqh, p.sqt, p.skb, p.skh, p.skt, p.svb, p.svh, p.svt, p.sob, p.soh, p.sot};
    for (long long x : s)
      if (x >= (1LL << 38)) return SDPA_ERR_UNSUPPORTED;
  }
  if (p.use_rel) {
    if (p.d != 64) return SDPA_ERR_UNSUPPORTED;
    const int kw = p.kw_n;
    if (!(kw == 14 || kw == 16 || kw == 32 || kw == 64)) return SDPA_ERR_UNSUPPORTED;
    if (p.kh_n > kRelHMax) return SDPA_ERR_UNSUPPORTED;
    // the padded tables borrow one K/V stage buffer: at most BN rows
    if (rel_rows_padded(p) > (kw == 14 ? 112 : 128)) return SDPA_ERR_UNSUPPORTED;
    if (!al16(p.rel_h) || !al16(p.rel_w)) return SDPA_ERR_MISALIGNED;
  }
  return SDPA_OK;
}

// Units (256-row query blocks of one (batch, head)) of a problem.
long long nblk_of(const Params& p, int nqblk) { return (long long)nqblk * p.Hq * p.B; }
// Key-tile width of the kernel instance the problem dispatches to.
// head_dim 128 with a mask tensor runs 64-key tiles with two S buffers per
// query tile (measured faster there: 3.32 ms against 3.97 ms on the 8192-token
// float-mask problem); without one, 128-key tiles (1.09 ms against 1.22 ms causal).
int BN_of(const Params& p) {
  if (p.use_rel) return p.kw_n == 14 ? 112 : 128;
  const bool tensor_mask = p.mask_kind == SDPA_MASK_ADD_FLOAT || p.mask_kind == SDPA_MASK_BOOL;
  return (p.d == 128 && tensor_mask) ? 64 : 128;
}

// Picks how many units run whole (first) and into how many parts each of the
// rest is split, minimising the modelled time on nsm SMs with one CTA each.
// A whole unit costs nt key tiles plus a fixed per-CTA cost (prologue,
// epilogue); a part costs its share of the tiles, the fixed cost, and the
// publish + merge of partial results.  Full waves of whole units go first and
// the remainder is split finely enough to fill the last wave.  Causal /
// sliding units differ in length and are not split.
void tc_schedule(long long units, int nt, int nsm, bool ranged, bool rel, int* n_full, int* n_split) {
  *n_full = (int)units;
  *n_split = 1;
  if (ranged || nt < 2 || units <= 0) return;
  // fixed costs in key tiles (B200: ~2 us of prologue + epilogue per CTA, ~4.5 us with
  // rel-pos projections; ~1.9 us per key tile of 2 x 128 rows at head_dim 64)
  const double c0 = rel ? 4.0 : 2.0, cs = 2.0;
  double best = (double)((units + nsm - 1) / nsm) * (nt + c0);
  const long long full_waves = units / nsm;
  for (long long fw = full_waves; fw >= 0 && fw >= full_waves - 1; --fw) {
    const long long F = fw * nsm, R = units - F;
    if (R <= 0) continue;
    for (int sp = 2; sp <= kMaxSplit && sp <= nt; ++sp) {
      const double waves_tail = (double)((R * sp + nsm - 1) / nsm);
      const double cost = (double)fw * (nt + c0) + waves_tail * ((nt + sp - 1) / sp + c0 + cs);
      if (cost < best - 1e-9) {
        best = cost;
        *n_full = (int)F;
        *n_split = sp;
      }
    }
  }
}

cudaError_t launch_tc(const Params& p, cudaStream_t stream) {
  TcArgs a;
  memset(&a, 0, sizeof(a));
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint64_t rowb = (uint64_t)p.d * 2;
  const int BN = BN_of(p);  // the K/V box must match the kernel instance's key tile
  // (head_dim, token, head, batch) views with the tensors' own strides (bhsd, bshd, ...)
  bool ok = make_tmap_4d(&a.tq, p.q, bf, p.d, p.Tq, p.Hq, p.B, 2 * p.sqt, 2 * p.sqh, 2 * p.sqb, 64, 128, true);
  ok = ok && make_tmap_4d(&a.tk, p.k, bf, p.d, p.Tkv, p.Hkv, p.B, 2 * p.skt, 2 * p.skh, 2 * p.skb, 64, BN, true);
  ok = ok && make_tmap_4d(&a.tv, p.v, bf, p.d, p.Tkv, p.Hkv, p.B, 2 * p.svt, 2 * p.svh, 2 * p.svb, 64, BN, true);
  if (p.use_rel) {
    a.rel_n = rel_rows_padded(p);
    const uint64_t nh = p.qh_n + p.kh_n - 1, nw = p.qw_n + p.kw_n - 1;
    ok = ok && make_tmap_3d(&a.trh, p.rel_h, bf, 2, p.d, nh, 1, rowb, rowb * nh, 64, a.rel_n, true);
    ok = ok && make_tmap_3d(&a.trw, p.rel_w, bf, 2, p.d, nw, 1, rowb, rowb * nw, 64, a.rel_n, true);
  }
  ok = ok && make_tmap_4d(&a.to, p.out, bf, p.d, p.Tq, p.Hq, p.B, 2 * p.sot, 2 * p.soh, 2 * p.sob, 64, 32, true);
  if (!ok) return cudaErrorInvalidValue;
  a.out = p.out;
  a.sob = p.sob; a.soh = p.soh; a.sot = p.sot;
  a.lse = p.lse;
  a.mask = p.mask;
  a.msb = p.msb; a.msh = p.msh; a.msq = p.msq;
  a.offset = p.offset; a.window = p.window;
  a.B = p.B; a.Hq = p.Hq; a.Hkv = p.Hkv; a.Tq = p.Tq; a.Tkv = p.Tkv; a.group = p.group;
  a.mask_kind = p.mask_kind;
  if (p.mask_kind == SDPA_MASK_ADD_FLOAT)
    a.mask_vec = al16(p.mask) && !(p.msb % 8) && !(p.msh % 8) && !(p.msq % 8);
  if (p.mask_kind == SDPA_MASK_BOOL)
    a.mask_vec = al16(p.mask) && !(p.msb % 16) && !(p.msh % 16) && !(p.msq % 16);
  a.scale_log2 = p.scale * kLog2e;
  a.qw_n = p.qw_n; a.kh_n = p.kh_n; a.kw_n = p.kw_n;
  a.err = p.err;
  const int nqblk = (p.Tq + 2 * kRowsPerTile - 1) / (2 * kRowsPerTile);
  const int mk = tc_mask_code(p);
  tc_schedule(nblk_of(p, nqblk), (p.Tkv + BN_of(p) - 1) / BN_of(p), num_sms(), mk == TC_RANGE, p.use_rel != 0,
              &a.n_full, &a.n_split);
  a.nqblk = nqblk;
  // causal: query blocks with the most key tiles first, so the short ones fill the tail
  a.reverse_q = (mk == TC_RANGE && p.mask_kind == SDPA_MASK_CAUSAL) ? 1 : 0;
  // a float / bool mask tensor broadcast over heads: every head of a query
  // block reads the same mask rows, so those heads run side by side
  a.head_fast = ((mk == TC_FLOAT || mk == TC_BOOL) && p.msh == 0 && p.Hq > 1) ? 1 : 0;
  a.fd_split = make_fastdiv((uint32_t)a.n_split);
  a.fd_hq = make_fastdiv((uint32_t)p.Hq);
  a.fd_nqblk = make_fastdiv((uint32_t)nqblk);
  a.fd_group = make_fastdiv((uint32_t)p.group);
  a.fd_qw = make_fastdiv((uint32_t)p.qw_n);
  const long long units = nblk_of(p, nqblk);
  const long long n_split_units = units - a.n_full;
  if (n_split_units > 0) {
    const size_t nml = (size_t)n_split_units * a.n_split * 256 * sizeof(float2);
    const size_t no = (size_t)n_split_units * a.n_split * 256 * p.d * sizeof(float);
    void *cnt = nullptr, *data = nullptr;
    if (workspace_get((size_t)n_split_units * sizeof(int), nml + no, &cnt, &data, stream) != SDPA_OK)
      return cudaErrorMemoryAllocation;
    a.ws_cnt = static_cast<int*>(cnt);
    a.ws_ml = static_cast<float2*>(data);
    a.ws_o = reinterpret_cast<float*>(static_cast<char*>(data) + nml);
  }
  dim3 grid((unsigned)(a.n_full + n_split_units * a.n_split), 1u, 1u);
  if (!p.use_rel) {
    if (p.d == 64) return dispatch_mask<64, 128, 0, 3>(mk, a, grid, stream);
    if (BN_of(p) == 64) {
      // a mask tensor whose rows TMA can read: mask tiles staged by TMA
      // (three K/V stages leave room for two mask stages per query tile)
      if ((mk == TC_FLOAT || mk == TC_BOOL) && a.mask_vec) {
        const uint64_t es = mk == TC_FLOAT ? 2 : 1;
        const uint64_t hm = p.msh ? (uint64_t)p.Hq : 1, bm = p.msb ? (uint64_t)p.B : 1;
        const uint64_t sq = es * (uint64_t)p.msq;
        const uint64_t sh = p.msh ? es * (uint64_t)p.msh : sq * (uint64_t)p.Tq;
        const uint64_t sb = p.msb ? es * (uint64_t)p.msb : sh * hm;
        const bool fl = mk == TC_FLOAT;
        if (make_tmap_4d(&a.tm, p.mask, fl ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, p.Tkv,
                         p.Tq, hm, bm, sq, sh, sb, 64, kRowsPerTile,
                         fl ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
          return fl ? launch_one<128, 64, 0, TC_FLOAT_TMA, 3>(a, grid, stream)
                    : launch_one<128, 64, 0, TC_BOOL_TMA, 3>(a, grid, stream);
      }
      return dispatch_mask<128, 64, 0, 4>(mk, a, grid, stream);
    }
    return dispatch_mask<128, 128, 0, 2>(mk, a, grid, stream);
  }
  switch (p.kw_n) {
    case 14: return dispatch_mask<64, 112, 14, 3>(mk, a, grid, stream);
    case 16: return dispatch_mask<64, 128, 16, 2>(mk, a, grid, stream);
    case 32: return dispatch_mask<64, 128, 32, 2>(mk, a, grid, stream);
    case 64: return dispatch_mask<64, 128, 64, 2>(mk, a, grid, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace sdpa
