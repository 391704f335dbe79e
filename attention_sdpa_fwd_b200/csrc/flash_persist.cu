// Persistent tensor-core SDPA forward for many short problems (sm_100a).
//
// Same computation as the tensor-core kernel in flash_tc.cu,
// softmax(Q.K^T*scale + bias).V with SAM's decomposed rel-pos bias built in
// the kernel (candle PR "SDPA with Relative Positional Embeddings": term_h /
// term_w added to the scores), for workloads made of many small attention
// problems.  SAM's windowed blocks attend inside each 14x14 window
// (mlx-examples issue "segment_anything: fuse attention with
// mx.fast.scaled_dot_product_attention": the windowed and global blocks share
// the attention call), so one (window, head) is 196 query rows against 196
// keys: two key tiles.  With one CTA per problem the fixed costs (Q load,
// rel-pos projections, output store, CTA launch) last as long as the work.
// Here one CTA per SM walks the units c, c + G, c + 2G, ... (a unit is one
// 256-row query block of one (batch, head)) and overlaps consecutive units:
//   * the next unit's Q tiles land in the second of two Q buffers while the
//     current unit runs;
//   * K/V tiles stream through one stage ring counted over all units;
//   * S_t of the next unit's first key tile is issued as soon as softmax t
//     has read the current unit's last S_t;
//   * the next unit's rel-pos projections Q_t.Rh^T and Q_t.Rw^T are computed
//     into the P_t columns right after the current unit's last P_t.V, and
//     softmax t scatters them to shared memory after its epilogue.
//
// Warp roles (384 threads): warps 0-3 softmax of query tile A (thread = row =
// TMEM lane), warps 4-7 tile B, warp 8 K/V producer (TMA), warp 9 TMEM owner
// and MMA issuer (one elected lane issues), warp 10 Q producer (TMA), warp 11 idle.
// TMEM: S_A [0,128) S_B [128,256) O_A [256,320) O_B [320,384) P_A [384,448)
// P_B [448,512); between units Ph_t = [384+64t, +32), Pw_t = [384+64t+32, +32).
//
// Every barrier phase is counted over the CTA's whole tile sequence
// g = it*nt + j (it-th unit of the CTA, key tile j of nt), so the
// per-unit hand-over needs no barrier of its own:
//   * P_t of a unit's first tile overwrites P_t(g-1) only after the epilogue
//     of the previous unit waited for O_t += P_t(g-1).V;
//   * the first P.V of a unit overwrites O_t (no accumulate) only after
//     softmax t read O_t out (its P arrival comes after its epilogue);
//   * the projections of unit it+1 overwrite the P columns after the last
//     P.V of unit it in issue order (tcgen05.mma from one thread execute in order).
#include <math.h>
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
constexpr int kRegsLaunch = 168;
// 216 + 72: the producer, Q-loader and MMA warps spill less than with 56
// registers (68 -> 16 spilled bytes), and the windowed SAM workload runs 7 %
// faster (65.3 -> 60.9 us); the softmax loop does not need more than 216 here.
constexpr int kRegsSoftmax = 216;
constexpr int kRegsOther = (kThreads * kRegsLaunch - 2 * 128 * kRegsSoftmax) / 128;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther <= kThreads * kRegsLaunch, "register split");
constexpr int kRows = 128;        // query rows per tile
constexpr int kD = 64;            // head_dim
constexpr int kRelH = 16;         // key-grid height limit: 2*16-1 table rows fit 32 TMEM columns
constexpr int kRelCols = 32;      // TMEM columns (and padded table rows) per projection
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: O is rescaled only when the max grows by 2^8

struct PsArgs {
  CUtensorMap tq, tk, tv, trh, trw;
  CUtensorMap to;  // out, 32-row boxes: each softmax warp stores its rows with one TMA store
  void* out;
  long long sob, soh, sot;
  float* lse;
  int Hq, Tq, Tkv, group;
  float scale_log2;
  int qw_n, kh_n;
  int nqblk;   // 256-row query blocks per (batch, head)
  int units;   // nqblk * Hq * B
  int* err;
  // the divisors of the unit decode, of the tile count and of the query grid,
  // as FastDiv (the CTA count is the grid's, fixed at launch)
  FastDiv fd_nqblk, fd_hq, fd_group, fd_nt, fd_qw, fd_grid;
};

template <int BN, int KW, int NS>
struct PLayout {
  static constexpr int kQBytes = kRows * 128;       // one 128-row Q tile (128 B rows, 128-B swizzle)
  static constexpr int kQBuf = 2 * kQBytes;         // both tiles of a unit
  static constexpr int kKVBytes = BN * 128;         // one K or V tile
  static constexpr int kTabBytes = kRelCols * 128;  // one padded rel table
  static constexpr int oQ = 0;
  static constexpr int oK = oQ + 2 * kQBuf;
  static constexpr int oV = oK + NS * kKVBytes;
  static constexpr int oTab = oV + NS * kKVBytes;
  static constexpr int oRel = oTab + (KW > 0 ? 2 * kTabBytes : 0);
  static constexpr int kRelRows = KW > 0 ? kRelH + KW : 0;  // rel_h rows then rel_w rows, 256 floats each
  static constexpr int oBar = oRel + kRelRows * 256 * 4;
  static constexpr int kBars = 4 * NS + 17;
  static constexpr int kTotal = oBar + kBars * 8 + 16;
  static constexpr int kAlloc = kTotal + 1024;  // slack for 1024-byte alignment
  static_assert(kAlloc <= 232448, "shared memory budget");
  static_assert(oK % 1024 == 0 && kKVBytes % 1024 == 0 && oTab % 1024 == 0, "swizzle atoms stay aligned");
  static_assert(KW == 0 || BN % (KW > 0 ? KW : 1) == 0, "key tile must hold whole key-grid rows");
};

struct UnitPos {
  int b, h, q0;
};

__device__ __forceinline__ UnitPos unit_pos(const PsArgs& a, int u) {
  UnitPos r;
  const int bh = (int)fdiv((uint32_t)u, a.fd_nqblk);
  r.q0 = (u - bh * a.nqblk) * 2 * kRows;
  r.b = (int)fdiv((uint32_t)bh, a.fd_hq);
  r.h = bh - r.b * a.Hq;
  return r;
}

template <int BN, int KW, int NS>
__global__ void __launch_bounds__(kThreads, 1) flash_fwd_persist(const __grid_constant__ PsArgs args) {
  using L = PLayout<BN, KW, NS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem + L::oQ;
  uint8_t* sK = smem + L::oK;
  uint8_t* sV = smem + L::oV;
  uint8_t* sTab = smem + L::oTab;
  float* sRel = reinterpret_cast<float*>(smem + L::oRel);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::oBar);
  uint64_t* k_full = bars;            // [NS] TMA -> MMA
  uint64_t* v_full = bars + NS;       // [NS]
  uint64_t* k_empty = bars + 2 * NS;  // [NS] MMA commit after both Q.K^T reading the stage -> TMA
  uint64_t* v_empty = bars + 3 * NS;  // [NS] MMA commit after both P.V reading the stage -> TMA
  uint64_t* q_full = bars + 4 * NS;   // [2]  Q buffer landed
  uint64_t* q_empty = q_full + 2;     // [2]  every MMA of the unit in that Q buffer issued and done
  uint64_t* s_full = q_full + 4;      // [2]  S_t ready (MMA commit)
  uint64_t* s_free = q_full + 6;      // [2]  softmax t read S_t (128 arrivals)
  uint64_t* p_full = q_full + 8;      // [2]  softmax t wrote P_t (128 arrivals)
  uint64_t* o_ready = q_full + 10;    // [2]  O_t += P_t.V done (MMA commit)
  uint64_t* rel_mma = q_full + 12;    // a unit's rel projections in TMEM (MMA commit, once per unit)
  uint64_t* tab_full = q_full + 13;   // rel tables landed (once)
  uint64_t* fin = q_full + 14;        // last commit before TMEM release
  uint64_t* o_drained = q_full + 15;  // [2]  the unit's O rows staged in that Q buffer stored (8 arrivals)
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + L::kBars);
  int* abort_flag = reinterpret_cast<int*>(tslot + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  // programmatic dependent launch, as in the tensor-core kernel: nothing
  // before grid_dep_wait() touches global memory
  grid_dep_launch();
  const int G = gridDim.x;
  const int n_units =
      (int)blockIdx.x < args.units ? (int)fdiv((uint32_t)(args.units - (int)blockIdx.x + G - 1), args.fd_grid) : 0;
  const int nt = (args.Tkv + BN - 1) / BN;
  const int total = n_units * nt;

  if (tid == 0) {
    *abort_flag = 0;
    for (int i = 0; i < L::kBars; ++i) mbar_init(&bars[i], 1);
    mbar_init(&s_free[0], kRows);
    mbar_init(&s_free[1], kRows);
    mbar_init(&p_full[0], kRows);
    mbar_init(&p_full[1], kRows);
    mbar_init(&o_drained[0], 8);
    mbar_init(&o_drained[1], 8);
    fence_mbar_init();
    grid_dep_wait();
    if (n_units > 0) {
      // the first unit's Q, the rel tables and K tile 0 go out before the
      // TMEM allocation and the CTA barrier
      tma_prefetch_desc(&args.tq);
      tma_prefetch_desc(&args.tk);
      if (KW > 0) {
        mbar_expect_tx(tab_full, 2 * L::kTabBytes);
        tma_load_3d(sTab, &args.trh, tab_full, 0, 0, 0);
        tma_load_3d(sTab + L::kTabBytes, &args.trw, tab_full, 0, 0, 0);
      }
      const UnitPos u0 = unit_pos(args, blockIdx.x);
      mbar_expect_tx(&q_full[0], 2 * L::kQBytes);
      for (int t = 0; t < 2; ++t)
        tma_load_4d(sQ + t * L::kQBytes, &args.tq, &q_full[0], 0, u0.q0 + t * kRows, u0.h, u0.b);
      mbar_expect_tx(&k_full[0], L::kKVBytes);
      tma_load_4d(sK, &args.tk, &k_full[0], 0, 0, (int)fdiv((uint32_t)u0.h, args.fd_group), u0.b);
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

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kRegsOther));
    if (warp == 8) {
      // ---------------------------------------------------------- K/V producer
      // K runs one tile ahead of V; stages are counted over all units, so the
      // next units' tiles are requested as soon as their stages free up.
      if (lane == 0 && n_units > 0) {
        tma_prefetch_desc(&args.tv);
        bool ok = true;
        int k_issued = 1, v_issued = 0;
        auto load_kv = [&](int g, bool is_k) {
          const int s = g % NS, use = g / NS;
          if (use > 0) ok = mbar_wait(is_k ? &k_empty[s] : &v_empty[s], (use - 1) & 1, abort_v, args.err);
          if (!ok) return;
          const int it = (int)fdiv((uint32_t)g, args.fd_nt);
          const UnitPos u = unit_pos(args, blockIdx.x + it * G);
          const int key0 = (g - it * nt) * BN;
          uint64_t* bar = is_k ? &k_full[s] : &v_full[s];
          mbar_expect_tx(bar, L::kKVBytes);
          tma_load_4d((is_k ? sK : sV) + s * L::kKVBytes, is_k ? &args.tk : &args.tv, bar, 0, key0,
                      (int)fdiv((uint32_t)u.h, args.fd_group), u.b);
          if (is_k) k_issued = g + 1; else v_issued = g + 1;
        };
        for (int g = 1; g < total && ok; ++g) {
          load_kv(g, true);
          if (ok) load_kv(g - 1, false);
        }
        if (ok) load_kv(total - 1, false);
        if (!ok) {
          // abandoned: let the copies already in flight land before the CTA exits
          for (int g = max(0, k_issued - NS); g < k_issued; ++g)
            mbar_wait(&k_full[g % NS], (g / NS) & 1, nullptr, args.err);
          for (int g = max(0, v_issued - NS); g < v_issued; ++g)
            mbar_wait(&v_full[g % NS], (g / NS) & 1, nullptr, args.err);
          if (KW > 0) mbar_wait(tab_full, 0, nullptr, args.err);
        }
      }
    } else if (warp == 10) {
      // ---------------------------------------------------------- Q producer
      // The Q tiles of unit it go into buffer it & 1 once every MMA of unit
      // it - 2 is done and the output rows unit it - 2 staged there are
      // stored (a warp of its own, so that waiting for that never holds back
      // the K/V stream).
      if (lane == 0 && n_units > 1) {
        bool ok = true;
        int q_issued = 1;
        for (int it = 1; it < n_units && ok; ++it) {
          const int qb = it & 1;
          if (it >= 2) ok = mbar_wait(&q_empty[qb], ((it >> 1) - 1) & 1, abort_v, args.err);
          if (ok && it >= 2) ok = mbar_wait(&o_drained[qb], ((it >> 1) - 1) & 1, abort_v, args.err);
          if (!ok) break;
          const UnitPos u = unit_pos(args, blockIdx.x + it * G);
          mbar_expect_tx(&q_full[qb], 2 * L::kQBytes);
          for (int t = 0; t < 2; ++t)
            tma_load_4d(sQ + qb * L::kQBuf + t * L::kQBytes, &args.tq, &q_full[qb], 0, u.q0 + t * kRows, u.h, u.b);
          q_issued = it + 1;
        }
        if (!ok) {
          for (int it = max(0, q_issued - 2); it < q_issued; ++it)
            mbar_wait(&q_full[it & 1], (it >> 1) & 1, nullptr, args.err);
        }
      }
    } else if (warp == 9) {
      // ---------------------------------------------------------- MMA issuer
      // The whole warp runs the loop (waits are warp-uniform) and one elected
      // lane issues each instruction.  Per tile g: S_A(g+1), O_A += P_A(g).V_g,
      // S_B(g+1), O_B += P_B(g).V_g; after a unit's last tile, the next unit's
      // projections.
      if (n_units > 0) {
        constexpr uint32_t id_qk = idesc_bf16_f32(128, BN, false, false);
        constexpr uint32_t id_pv = idesc_bf16_f32(128, kD, false, true);
        // both tables stacked as one 64-row operand: Ph_t and Pw_t come out of
        // one MMA per k-step into the 64 P_t columns
        constexpr uint32_t id_rel = idesc_bf16_f32(128, 2 * kRelCols, false, false);
        const uint64_t dq = sdesc_sw128(smem_u32(sQ), 16, 1024);
        const uint64_t dk = sdesc_sw128(smem_u32(sK), 16, 1024);
        const uint64_t dv = sdesc_sw128(smem_u32(sV), BN * 128, 1024);
        const uint64_t dtab = sdesc_sw128(smem_u32(sTab), 16, 1024);
        auto wait = [&](uint64_t* bar, uint32_t parity) {
          return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_v, args.err));
        };
        // descriptors are built once; a byte offset inside shared memory is
        // added to the start-address field (address >> 4)
        auto qk = [&](int t, int qb, int s) {
          const uint64_t a0 = dq + (uint64_t)((qb * L::kQBuf + t * L::kQBytes) >> 4);
          const uint64_t b0 = dk + (uint64_t)((s * L::kKVBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) mma_ss_w(tbase + t * 128, a0 + kk * 2, b0 + kk * 2, id_qk, kk > 0);
        };
        auto pv = [&](int t, int s, bool first) {
          const uint64_t b0 = dv + (uint64_t)((s * L::kKVBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            mma_ts_w(tbase + 256 + t * kD, tbase + 384 + t * 64 + kk * 8, b0 + (uint64_t)((kk * 16 * 128) >> 4),
                     id_pv, (!first) || kk > 0);
        };
        auto rel = [&](int qb) {
#pragma unroll
          for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk)
              mma_ss_w(tbase + 384 + t * 64, dq + (uint64_t)((qb * L::kQBuf + t * L::kQBytes + kk * 32) >> 4),
                       dtab + (uint64_t)((kk * 32) >> 4), id_rel, kk > 0);
          mma_commit_w(rel_mma);
        };
        bool ok = wait(&q_full[0], 0);
        if (ok && KW > 0) {
          ok = wait(tab_full, 0);
          if (ok) {
            tc_fence_after();
            rel(0);
          }
        }
        if (ok) ok = wait(&k_full[0], 0);
        if (ok) {
          tc_fence_after();
          qk(0, 0, 0);
          mma_commit_w(&s_full[0]);
          qk(1, 0, 0);
          mma_commit_w(&s_full[1]);
          mma_commit_w(&k_empty[0]);
        }
        for (int g = 0; g < total && ok; ++g) {
          const int it = (int)fdiv((uint32_t)g, args.fd_nt), j = g - it * nt, s = g % NS;
          const int g1 = g + 1;
          const bool more = g1 < total;
          const int it1 = (int)fdiv((uint32_t)g1, args.fd_nt), j1 = g1 - it1 * nt, s1 = g1 % NS, qb1 = it1 & 1;
          if (more) {
            if (j1 == 0) ok = wait(&q_full[qb1], (it1 >> 1) & 1);
            if (ok) ok = wait(&k_full[s1], (g1 / NS) & 1);
            if (ok) ok = wait(&s_free[0], g & 1);
            if (!ok) break;
            tc_fence_after();
            qk(0, qb1, s1);
            mma_commit_w(&s_full[0]);
          }
          ok = wait(&v_full[s], (g / NS) & 1);
          if (ok) ok = wait(&p_full[0], g & 1);
          if (!ok) break;
          tc_fence_after();
          pv(0, s, j == 0);
          mma_commit_w(&o_ready[0]);
          if (more) {
            ok = wait(&s_free[1], g & 1);
            if (!ok) break;
            tc_fence_after();
            qk(1, qb1, s1);
            mma_commit_w(&s_full[1]);
            mma_commit_w(&k_empty[s1]);
          }
          ok = wait(&p_full[1], g & 1);
          if (!ok) break;
          tc_fence_after();
          pv(1, s, j == 0);
          mma_commit_w(&o_ready[1]);
          mma_commit_w(&v_empty[s]);
          if (j == nt - 1) {
            // unit it is fully issued: the next unit's projections go into the
            // P columns, then unit it's Q buffer is released
            if (more && KW > 0) rel(qb1);
            mma_commit_w(&q_empty[it & 1]);
          }
        }
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kRegsSoftmax));
    // ------------------------------------------------------------ softmax of tile t
    const int t = warp >> 2;
    const int row = t * kRows + (warp & 3) * 32 + lane;  // row within the unit's 256-row block
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_addr = tbase + lane_off + t * 128;
    const uint32_t o_addr = tbase + lane_off + 256 + t * kD;
    const uint32_t p_addr = tbase + lane_off + 384 + t * 64;
    float* relh_s = sRel;               // [kRelH][256]
    float* relw_s = sRel + kRelH * 256;  // [KW][256]
    constexpr int NG = KW > 0 ? BN / KW : 1;  // key-grid rows per key tile
    constexpr int GW = BN / NG;               // keys per group
    static_assert(GW % 2 == 0, "groups hold whole pairs");
    const uint64_t sl2 = f2(args.scale_log2, args.scale_log2);
    bool ok = true;

    for (int it = 0; it < n_units && ok; ++it) {
      const UnitPos u = unit_pos(args, blockIdx.x + it * G);
      const long long qi = (long long)u.q0 + row;
      // (debug builds: the unit's batch and head lie inside the problem)
      const bool row_valid = qi < args.Tq && dcheck(args.err, qi >= 0 && u.h >= 0 && u.h < args.Hq &&
                                                                  ((long long)u.b * args.Hq + u.h) * args.nqblk < args.units);

      // this unit's rel_h / rel_w (log2 e prescaled): projections from the P
      // columns into this row's shared-memory slots; rel_w then in registers
      float rw[KW > 0 ? KW : 2];
      if constexpr (KW > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(rel_mma, it & 1, abort_v, args.err));
        if (!ok) break;
        tc_fence_after();
        const int qh = (int)fdiv((uint32_t)qi, args.fd_qw), qw = (int)qi - qh * args.qw_n, kh_n = args.kh_n;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          uint32_t r[32];
          tmem_ld32(p_addr + w * kRelCols, r);
          tmem_wait_ld();
          const int base_idx = w == 0 ? qh + kh_n - 1 : qw + KW - 1;
          const int nk = w == 0 ? kh_n : KW;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int k = base_idx - i;  // key-grid coordinate reached through table row i
            if (k >= 0 && k < nk && dcheck_idx(args.err, k, w == 0 ? kRelH : KW))
              (w == 0 ? relh_s : relw_s)[k * 256 + row] = __uint_as_float(r[i]) * kLog2e;
          }
        }
#pragma unroll
        for (int c = 0; c < KW; ++c) rw[c] = relw_s[c * 256 + row];
      }

      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < nt && ok; ++j) {
        const int g = it * nt + j;
        const int j0 = j * BN;
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[t], g & 1, abort_v, args.err));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[BN];
#pragma unroll
        for (int c0 = 0; c0 < BN; c0 += 32) {
          if (c0 + 32 <= BN)
            tmem_ld32p(s_addr + c0, sr + c0);
          else
            tmem_ld16p(s_addr + c0, sr + c0);
        }
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&s_free[t]);

        // x = s*scale (+ rel_w) in log2 units, two columns per instruction;
        // rel_h is constant over a key-grid row: kept per group (goff) and
        // folded into the max and the exponent
        uint64_t x2[BN / 2];
        float goff[NG];
        if constexpr (KW > 0) {
          const int kh0 = j0 / KW;
#pragma unroll
          for (int gi = 0; gi < NG; ++gi) {
            const int khi = kh0 + gi;
            goff[gi] = khi < args.kh_n ? relh_s[khi * 256 + row] : 0.f;
          }
#pragma unroll
          for (int gi = 0; gi < NG; ++gi)
#pragma unroll
            for (int c = 0; c < KW; c += 2) {
              const int e = gi * KW + c;
              x2[e / 2] = f2_fma(f2u(sr[e], sr[e + 1]), sl2, f2(rw[c], rw[c + 1]));
            }
        } else {
          goff[0] = 0.f;
#pragma unroll
          for (int i = 0; i < BN / 2; ++i) x2[i] = f2_mul(f2u(sr[2 * i], sr[2 * i + 1]), sl2);
        }
        if (j0 + BN > args.Tkv) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (j0 + c >= args.Tkv) {
              float lo, hi;
              f2_split(x2[c / 2], lo, hi);
              if (c & 1) hi = -INFINITY; else lo = -INFINITY;
              x2[c / 2] = f2(lo, hi);
            }
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
        // p = 2^(x + goff - m) packed to bf16 pairs in registers, so that the
        // wait for the previous P.V comes after the exponentials
        const float m_use = m_run == -INFINITY ? 0.f : m_run;
        uint32_t pk[BN / 2];
        l_run += tile::exp_pack<BN, GW>(x2, goff, m_use, pk);
        // O_t += P_t(g-1).V must be complete before O_t is rescaled or P_t
        // overwritten (for a unit's first tile the previous epilogue waited)
        if (j > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(&o_ready[t], (g - 1) & 1, abort_v, args.err));
          if (!ok) break;
          tc_fence_after();
        }
        if (j > 0 && __any_sync(0xffffffffu, need)) tile::rescale_o<kD>(o_addr, alpha);  // O_t row *= alpha
        tile::store_p<BN>(p_addr, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[t]);
      }
      if (!ok) break;

      // epilogue: O / l -> bf16 rows staged in this unit's Q tile t (its last
      // Q.K^T, which this warp waited for, was the tile's last reader), then
      // one TMA store of the warp's 32 rows (rows past Tq are not written);
      // the Q loader refills the buffer once every warp's store has read it
      ok = __all_sync(0xffffffffu, mbar_wait(&o_ready[t], (it * nt + nt - 1) & 1, abort_v, args.err));
      if (!ok) break;
      tc_fence_after();
      uint8_t* stage = sQ + (it & 1) * L::kQBuf + t * L::kQBytes + (warp & 3) * 32 * 128;
      tile::stage_o_row_sw128<kD>(o_addr, l_run > 0.f ? 1.f / l_run : 0.f, stage + lane * 128, lane, 0);
      fence_proxy_async_shared();
      __syncwarp();
      if (lane == 0) {
        const int r0 = u.q0 + t * kRows + (warp & 3) * 32;
        if (r0 < args.Tq) {
          tma_store_4d(&args.to, stage, 0, r0, u.h, u.b);
          bulk_commit();
          bulk_wait_read_all();
        }
        mbar_arrive(&o_drained[it & 1]);
      }
      if (row_valid && args.lse)
        args.lse[((long long)u.b * args.Hq + u.h) * args.Tq + qi] =
            l_run > 0.f ? m_run * kLn2 + logf(l_run) : -INFINITY;
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) {
    if (lane == 0 && n_units > 0) {
      // nothing this CTA issued may still be writing TMEM when it is released
      mma_commit(fin);
      mbar_wait(fin, 0, nullptr, args.err);
    }
    __syncwarp();
    tmem_dealloc(tbase, 512);
  }
}

template <int BN, int KW, int NS>
cudaError_t launch_persist_one(const PsArgs& a, int grid, cudaStream_t stream) {
  using L = PLayout<BN, KW, NS>;
  auto kern = flash_fwd_persist<BN, KW, NS>;
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
  // programmatic serialization (the kernel waits for the previous grid before
  // it touches global memory)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
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

bool al16p(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

// Whether the persistent kernel takes this problem: everything the tensor-core
// kernel takes at head_dim 64 without a mask, with rel-pos key-grid width 14
// or 16 and height up to 16 (both projections then fit the P columns), or
// without rel-pos.
int tc_persist_check(const Params& p, sdpa_dtype_t dtype) {
  const int rc = tc_check(p, dtype);
  if (rc != SDPA_OK) return rc;
  if (p.d != 64 || p.mask_kind != SDPA_MASK_NONE) return SDPA_ERR_UNSUPPORTED;
  if (p.use_rel) {
    if (!(p.kw_n == 14 || p.kw_n == 16)) return SDPA_ERR_UNSUPPORTED;
    if (p.kh_n > kRelH) return SDPA_ERR_UNSUPPORTED;
    // each table (Qh + Kh - 1, Qw + Kw - 1 rows) within its 32 projection columns
    if (p.qh_n + p.kh_n - 1 > kRelCols || p.qw_n + p.kw_n - 1 > kRelCols) return SDPA_ERR_UNSUPPORTED;
  }
  if (!al16p(p.out)) return SDPA_ERR_MISALIGNED;
  return SDPA_OK;
}

// Key tile of the persistent instance the problem dispatches to.
static int persist_bn(const Params& p) { return (p.use_rel && p.kw_n == 14) ? 112 : 128; }

// AUTO takes the persistent form for many short problems: at least two units
// per SM, each of at most four key tiles (there the fixed per-CTA costs are
// comparable to the work; longer problems keep the split schedule).
bool tc_persist_preferred(const Params& p) {
  const long long nqblk = (p.Tq + 2 * kRows - 1) / (2 * kRows);
  const long long units = nqblk * p.Hq * p.B;
  const int nt = (p.Tkv + persist_bn(p) - 1) / persist_bn(p);
  return units >= 2LL * num_sms() && nt <= 4;
}

cudaError_t launch_tc_persist(const Params& p, cudaStream_t stream) {
  PsArgs a;
  memset(&a, 0, sizeof(a));
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint64_t rowb = (uint64_t)p.d * 2;
  const int BN = persist_bn(p);
  bool ok = make_tmap_4d(&a.tq, p.q, bf, p.d, p.Tq, p.Hq, p.B, 2 * p.sqt, 2 * p.sqh, 2 * p.sqb, 64, kRows, true);
  ok = ok && make_tmap_4d(&a.tk, p.k, bf, p.d, p.Tkv, p.Hkv, p.B, 2 * p.skt, 2 * p.skh, 2 * p.skb, 64, BN, true);
  ok = ok && make_tmap_4d(&a.tv, p.v, bf, p.d, p.Tkv, p.Hkv, p.B, 2 * p.svt, 2 * p.svh, 2 * p.svb, 64, BN, true);
  ok = ok && make_tmap_4d(&a.to, p.out, bf, p.d, p.Tq, p.Hq, p.B, 2 * p.sot, 2 * p.soh, 2 * p.sob, 64, 32, true);
  if (p.use_rel) {
    // 32-row boxes (Qh + Kh - 1 <= 32 table rows); rows past a table read as zero
    const uint64_t nh = p.qh_n + p.kh_n - 1, nw = p.qw_n + p.kw_n - 1;
    ok = ok && make_tmap_3d(&a.trh, p.rel_h, bf, 2, p.d, nh, 1, rowb, rowb * nh, 64, kRelCols, true);
    ok = ok && make_tmap_3d(&a.trw, p.rel_w, bf, 2, p.d, nw, 1, rowb, rowb * nw, 64, kRelCols, true);
  }
  if (!ok) return cudaErrorInvalidValue;
  a.out = p.out;
  a.sob = p.sob; a.soh = p.soh; a.sot = p.sot;
  a.lse = p.lse;
  a.Hq = p.Hq; a.Tq = p.Tq; a.Tkv = p.Tkv; a.group = p.group;
  a.scale_log2 = p.scale * kLog2e;
  a.qw_n = p.qw_n; a.kh_n = p.kh_n;
  a.err = p.err;
  a.nqblk = (p.Tq + 2 * kRows - 1) / (2 * kRows);
  const long long units = (long long)a.nqblk * p.Hq * p.B;
  if (units > 0x7fffffffLL) return cudaErrorInvalidValue;
  a.units = (int)units;
  const int grid = (int)(units < num_sms() ? units : num_sms());
  a.fd_nqblk = make_fastdiv((uint32_t)a.nqblk);
  a.fd_hq = make_fastdiv((uint32_t)p.Hq);
  a.fd_group = make_fastdiv((uint32_t)p.group);
  a.fd_nt = make_fastdiv((uint32_t)((p.Tkv + persist_bn(p) - 1) / persist_bn(p)));
  a.fd_qw = make_fastdiv((uint32_t)p.qw_n);
  a.fd_grid = make_fastdiv((uint32_t)(grid > 0 ? grid : 1));
  if (!p.use_rel) return launch_persist_one<128, 0, 4>(a, grid, stream);
  if (p.kw_n == 14) return launch_persist_one<112, 14, 4>(a, grid, stream);
  return launch_persist_one<128, 16, 3>(a, grid, stream);
}

}  // namespace sdpa
