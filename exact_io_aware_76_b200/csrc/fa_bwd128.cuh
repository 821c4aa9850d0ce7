// fa_bwd128.cuh -- the backward's main kernel for head dim 128 on sm_100a: a CTA takes one or several 128-key
// tiles of one (batch, K/V head) in turn and walks 128-query tiles for each, so that every tcgen05 product has
// N = 128; with several, one tile's tail (last products, dK/dV store, last dQ reductions) overlaps the next
// one's loads and first products (barrier phases and the Q/dO ring run on across tiles).
//
// What it computes is the chain rule of O = softmax(scale * Q K^T + mask) V with P recomputed from the saved
// LSE (tiling plus recomputation: refbase entity page "FlashAttention", section "Capability"), per key tile
// and query tile:
//   S^T = K Q^T,  P^T = 2^(S^T c - LSE2)  (c = scale * log2 e, LSE2 = LSE * log2 e)
//   dP^T = V dO^T,  dS^T = P^T (dP^T - D)  (D_i = rowsum(dO_i * O_i), from the preprocess kernel)
//   dV += P^T dO,  dK += dS^T Q  (times scale at the end),  dQ^T partial = K^T dS^T  (fp32 reductions)
//
// Why 128 queries per tile: an M = 128 tcgen05 MMA with N = 64 occupies the tensor core as long as one with
// N = 128 (measured on B200: 64-72 cycles either way for K = 16), so the 64-query tiles that double-buffered
// S^T / dP^T in TMEM ran three of the five products at half rate. Here every product is 128 x 128 x 128.
//
// TMEM (512 columns): dV [0,128), dK [128,256), RS [256,384) = S^T then P^T (16-bit, packed in pairs; the
// warpgroup for queries 64h..64h+63 writes its P^T over the first 32 of its own 64 S^T columns), RP [384,512) =
// dP^T then the tile's dQ^T partial (lane = head-dim index, column = query).
// Shared memory: K, V (static), Q and dO in a 2-stage ring, dS^T (keys x queries, two 64-query 128-byte
// swizzled chunks): the A operand of dK (K-major) and the B operand of dQ^T (MN-major).
//
// Warps: 0-7 compute (thread = key row = TMEM lane; warpgroup h = warps 4h..4h+3 owns query columns
// 64h..64h+63 of every tile), 8-11 dQ (lane = head-dim index: TMEM -> registers -> red.global.add.v4 into
// the fp32 accumulator), 12 TMA, 13 TMEM allocation and MMA issue, 14-15 idle (their registers go to the
// others). MMA issue order per tile, so that the compute warps' exponentials overlap dK/dQ of the previous tile
// and dP of this one:
//   ... [P_i ready] dV_i, S_{i+1} | [dS_i ready] dK_i, dQ^T_i | [dQ^T_i read out] dP_{i+1} | [P_{i+1}] dV_{i+1} ...
// dQ accumulator layout (fp32, caller workspace): [B, H, Sq_pad / 4, 128, 4] -- four consecutive queries of one
// head-dim index are 16 contiguous bytes, so a warp's reduction for four queries covers 512 contiguous bytes.
#pragma once
#include "fa_bwd.cuh"

namespace fa {

struct Bwd128Smem {
  static constexpr int kBQ = 128, kNQS = 2;
  static constexpr int kTile = 128 * 128 * 2;  // one 128-row tile of K, V, Q, dO or dS^T (two 16 KB chunks)
  // Header at the start of the dynamic shared memory: barriers, TMEM address, abort flag, LSE2 and D per stage.
  static constexpr int kNumBars = 14;
  static constexpr int kBarOff = 0;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;   // TMEM address, abort flag
  static constexpr int kLOff = 128;                         // LSE2 per stage, 128 floats
  static constexpr int kDVecOff = kLOff + kNQS * kBQ * 4;    // D per stage, 128 floats
  static constexpr int kHeader = kDVecOff + kNQS * kBQ * 4;  // 2176 bytes
  // Tile area, 1024-byte aligned (128-byte swizzle atoms): K, V, Q[2], dO[2], dS^T.
  static constexpr int kKOff = 0, kVOff = kTile, kQOff = 2 * kTile, kDOOff = 4 * kTile, kDSOff = 6 * kTile;
  static constexpr int kTiles = 7 * kTile;  // 229376
  // The per-block maximum of dynamic shared memory on sm_100: a 1024-aligned window (the usual case) holds the
  // header rounded up to 1024 plus the tiles exactly; the kernel checks and refuses otherwise.
  static constexpr int kAlloc = 232448;
  static constexpr uint32_t kColDV = 0, kColDK = 128, kColS = 256, kColP = 384, kTmemCols = 512;
  static constexpr int kThreads = 512;
  // 512 x 128 registers at launch; compute and dQ warpgroups 144, the TMA/MMA warpgroup 80:
  // 3 * 128 * 144 + 128 * 80 = 65536 (neither side spills at this split).
  static constexpr uint32_t kRegsWork = 144, kRegsOther = 80;
};

// An empty asm that claims to modify two 64-bit values: the compiler must assume they change here, so it derives
// the per-instruction descriptors from them where they are used instead of keeping all of them live.
__device__ __forceinline__ void opaque(uint64_t& a, uint64_t& b) { asm volatile("" : "+l"(a), "+l"(b)); }

template <bool kBF16, bool kCausal, bool kDrop = false>
__global__ void __launch_bounds__(512, 1)
    fa_bwd_main128_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                          const BwdParams p) {
  using L = Bwd128Smem;
  constexpr int BQ = L::kBQ, NQS = L::kNQS;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t tiles_u32 = (raw_u32 + L::kHeader + 1023u) & ~1023u;
  if (tiles_u32 + L::kTiles > raw_u32 + L::kAlloc) {
    // The dynamic shared memory window is not 1024-byte aligned, so the tiles would not fit: refuse (uniformly,
    // before any barrier, copy or TMEM allocation) rather than run past the allocation.
    if (threadIdx.x == 0) atomicExch(&g_device_status, FA_ERR_UNSUPPORTED);
    return;
  }
  uint8_t* smem = smem_raw + (tiles_u32 - raw_u32);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + L::kBarOff);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;   // [NQS] Q, dO, LSE2, D of a stage arrived
  uint64_t* q_empty = bars + 3;  // [NQS] dK (the stage's last reader) done
  uint64_t* s_full = bars + 5;   // S^T in RS
  uint64_t* dp_full = bars + 6;  // dP^T in RP
  uint64_t* p_ready = bars + 7;  // P^T in RS, S^T read (256 compute threads)
  uint64_t* ds_ready = bars + 8; // dS^T in shared memory, dP^T read (256 compute threads)
  uint64_t* dq_full = bars + 9;  // dQ^T partial in RP
  uint64_t* dq_empty = bars + 10;  // dQ^T partial read out (128 dQ threads)
  uint64_t* ds_empty = bars + 11;  // dK and dQ^T done with the dS^T buffer
  uint64_t* dkv_done = bars + 12;  // a unit's products complete (dK/dV readable, K/V reloadable)
  uint64_t* mma_drain = bars + 13; // every product complete (before TMEM is released)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem_raw + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem_raw + L::kMiscOff + 4);

  // Work: a CTA owns p.units key tiles ("units") of one (batch, K/V head) and walks them one after the other,
  // each with every query head of the group, accumulating that tile's dK/dV in TMEM, so that one unit's tail
  // (its last products, the dK/dV store, the last dQ reductions) overlaps the next one's loads and first
  // products instead of a CTA exit and a new CTA's setup. For the causal mask the key tiles are dealt
  // alternately from both ends (0, n-1, 1, n-2, ...), so every CTA gets about the same number of query tiles.
  // CTA order: head-major for large problems (the units of one (batch, K/V head) together), so that its Q, dO
  // and dQ accumulator stay in L2; otherwise across heads. With one unit per CTA the key tiles run heavy-first.
  const int n_bh = p.B * p.Hkv;
  const int bh = p.head_major ? blockIdx.x / p.n_grp : blockIdx.x % n_bh;
  const int grp = p.head_major ? blockIdx.x % p.n_grp : blockIdx.x / n_bh;
  const int b = bh / p.Hkv, h_kv = bh % p.Hkv;
  const int off = p.Sk - p.Sq;
  const int n_units = max(0, min(p.units, p.n_kblk - grp * p.units));
  // Query r sees key j iff r + off - left <= j <= r + off + right (causal caps right at 0; negative bounds are
  // unbounded), i.e. j - off - right <= r <= j - off + left.
  const bool has_left = p.win_left >= 0;
  const int right = kCausal ? (p.win_right >= 0 ? min(p.win_right, 0) : 0) : p.win_right;
  const bool has_right = right >= 0;
  // Unit u: key tile, its query tiles [i_begin, i_begin + n_q) per head, n_it = n_q * group iterations
  // (iteration it: head it / n_q).
  struct Unit {
    int key0, i_begin, n_q, n_it;
  };
  auto unit_at = [&](int u) {
    const int i = grp * p.units + u;
    const int kblk = p.units == 1 ? i : ((i & 1) ? p.n_kblk - 1 - i / 2 : i / 2);
    Unit U;
    U.key0 = kblk * 128;
    const int key1 = min(p.Sk - 1, U.key0 + 127);
    const int r_min = has_right ? max(0, U.key0 - off - right) : 0;
    const int r_max = has_left ? min(p.Sq - 1, key1 - off + p.win_left) : p.Sq - 1;
    U.i_begin = r_min / BQ;
    U.n_q = (r_max >= r_min) ? r_max / BQ - U.i_begin + 1 : 0;
    U.n_it = U.n_q * p.group;
    return U;
  };

  const uint32_t warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < NQS; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_ready, 256);
    mbar_init(ds_ready, 256);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, 128);
    mbar_init(ds_empty, 1);
    mbar_init(dkv_done, 1);
    mbar_init(mma_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 13) {
    tmem_alloc(tmem_holder, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_holder;

  if (warp >= 12) {
    regs_dec<L::kRegsOther>();
    if (warp == 12 && lane == 0 && n_units > 0) {
      // ---------------------------------------------------------------- TMA producer
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      int nq = 0;  // Q/dO loads issued
      // Q, dO, LSE2 and D of global iteration gi (counted over this CTA's units) into stage gi % NQS.
      auto load_q = [&](int gi, const Unit& U, int it) -> bool {
        const int s = gi % NQS;
        const int h = h_kv * p.group + it / U.n_q;
        const int q0 = (U.i_begin + it % U.n_q) * BQ;
        const size_t row0 = (static_cast<size_t>(b) * p.H + h) * p.Sq_pad + q0;
        if (gi >= NQS && !mbar_wait(&q_empty[s], ((gi / NQS) - 1) & 1, abort_flag)) return false;
        mbar_arrive_expect_tx(&q_full[s], 2 * L::kTile + 2 * BQ * 4);
        for (int c = 0; c < 2; ++c) {
          tma_load_4d(smem + L::kQOff + s * L::kTile + c * 16384, &tm_q, &q_full[s], 64 * c, h, q0, b);
          tma_load_4d(smem + L::kDOOff + s * L::kTile + c * 16384, &tm_do, &q_full[s], 64 * c, h, q0, b);
        }
        bulk_load(smem_raw + L::kLOff + s * BQ * 4, p.lse2 + row0, BQ * 4, &q_full[s]);
        bulk_load(smem_raw + L::kDVecOff + s * BQ * 4, p.dvec + row0, BQ * 4, &q_full[s]);
        ++nq;
        return true;
      };
      int g = 0, w = 0;  // iterations issued, units with work loaded
      bool ok = true;
      for (int u = 0; ok && u < n_units; ++u) {
        const Unit U = unit_at(u);
        if (U.n_it == 0) continue;
        // The unit's first Q/dO tile only needs its ring stage; K and V wait until every product of the
        // previous unit (the last readers of the K/V buffers) is complete.
        if (!load_q(g, U, 0)) { ok = false; break; }
        if (w > 0 && !mbar_wait(dkv_done, (w - 1) & 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(kv_full, 2 * L::kTile);
        for (int c = 0; c < 2; ++c) {
          tma_load_4d(smem + L::kKOff + c * 16384, &tm_k, kv_full, 64 * c, h_kv, U.key0, b);
          tma_load_4d(smem + L::kVOff + c * 16384, &tm_v, kv_full, 64 * c, h_kv, U.key0, b);
        }
        ++w;
        ++g;
        for (int it = 1; it < U.n_it; ++it, ++g)
          if (!load_q(g, U, it)) { ok = false; break; }
      }
      if (*abort_flag) {
        // Let the copies already issued land before the CTA exits (bounded; own flag).
        int drain = 0;
        if (w > 0) mbar_wait(kv_full, (w - 1) & 1, &drain);
        for (int jj = max(0, nq - NQS); jj < nq; ++jj) {
          drain = 0;
          mbar_wait(&q_full[jj % NQS], (jj / NQS) & 1, &drain);
        }
      }
    } else if (warp == 13 && lane == 0 && n_units > 0) {
      // ---------------------------------------------------------------- MMA issuer
      constexpr uint32_t id_kk = idesc_f16(kBF16, 128, 128, false, false);  // S^T, dP^T: A, B K-major
      constexpr uint32_t id_kv = idesc_f16(kBF16, 128, 128, false, true);   // dV (A in TMEM), dK: B MN-major
      constexpr uint32_t id_q = idesc_f16(kBF16, 128, 128, true, true);     // dQ^T = K^T dS^T: both MN-major
      // One descriptor per buffer; each MMA adds a compile-time byte offset (plus a stage offset).
      const uint32_t k_base = smem_u32(smem + L::kKOff), v_base = smem_u32(smem + L::kVOff);
      const uint32_t q_base = smem_u32(smem + L::kQOff), do_base = smem_u32(smem + L::kDOOff);
      const uint32_t ds_base = smem_u32(smem + L::kDSOff);
      const uint64_t k_kmaj = sdesc_sw128(k_base, 16, 1024), v_kmaj = sdesc_sw128(v_base, 16, 1024);
      const uint64_t k_mn = sdesc_sw128(k_base, 16384, 1024);
      const uint64_t q_kmaj = sdesc_sw128(q_base, 16, 1024), do_kmaj = sdesc_sw128(do_base, 16, 1024);
      const uint64_t q_mn = sdesc_sw128(q_base, 16384, 1024), do_mn = sdesc_sw128(do_base, 16384, 1024);
      const uint64_t ds_kmaj = sdesc_sw128(ds_base, 16, 1024), ds_mn = sdesc_sw128(ds_base, 16384, 1024);
      // S^T = K Q^T (into RS) and dP^T = V dO^T (into RP): K-major operands, head dim advanced 16 elements
      // (32 bytes) per instruction, 64-element chunks 16 KB apart.
      // (opaque() keeps the compiler from precomputing every instruction's descriptor for the whole loop,
      // which would not fit in this warp's registers; the adds are a few integer instructions per MMA.)
      auto issue_s = [&](int it) {
        uint64_t a = k_kmaj, bq = sdesc_add(q_kmaj, (it % NQS) * L::kTile);
        opaque(a, bq);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t o = (kk / 4) * 16384 + (kk % 4) * 32;
          umma_ss(tmem + L::kColS, sdesc_add(a, o), sdesc_add(bq, o), id_kk, kk > 0);
        }
      };
      auto issue_dp = [&](int it) {
        uint64_t a = v_kmaj, bq = sdesc_add(do_kmaj, (it % NQS) * L::kTile);
        opaque(a, bq);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t o = (kk / 4) * 16384 + (kk % 4) * 32;
          umma_ss(tmem + L::kColP, sdesc_add(a, o), sdesc_add(bq, o), id_kk, kk > 0);
        }
      };
      bool ok = true;
      int g = 0, w = 0;  // global iteration, units with work
      for (int u = 0; ok && u < n_units; ++u) {
        const Unit U = unit_at(u);
        if (U.n_it == 0) continue;
        const int n_it = U.n_it;
        // The unit's first S^T and dP^T: RS is free once the previous unit's last dV (issued before, so it
        // executes before) has read P^T; RP once the dQ warps have read the previous unit's last dQ^T out.
        ok = mbar_wait(kv_full, w & 1, abort_flag) && mbar_wait(&q_full[g % NQS], (g / NQS) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after_sync();
        issue_s(g);
        umma_commit(s_full);
        if (g > 0 && !mbar_wait_spin(dq_empty, (g - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after_sync();
        issue_dp(g);
        umma_commit(dp_full);
        for (int it = 0; it < n_it; ++it) {
          const int gi = g + it;
          const int s = gi % NQS;
          const bool more = it + 1 < n_it;
          // dV += P^T dO: A = P^T from TMEM (16 queries = 8 columns per instruction; queries 64h.. start at
          // column 64h of RS), B = dO MN-major (16 query rows = 2048 bytes per instruction). The unit's first
          // dV overwrites the accumulator: its P_ready also says that the compute warps have read the previous
          // unit's dV and dK out of TMEM.
          if (!mbar_wait(p_ready, gi & 1, abort_flag)) { ok = false; break; }
          tc_fence_after_sync();
          {
            uint64_t dod = sdesc_add(do_mn, s * L::kTile), unused = 0;
            opaque(dod, unused);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_ts(tmem + L::kColDV, tmem + L::kColS + (kk / 4) * 64 + (kk % 4) * 8, sdesc_add(dod, kk * 2048),
                      id_kv, (it > 0 || kk > 0));
          }
          // The next tile's S^T can follow at once: its P^T was read by the dV product just issued (the tensor
          // core executes in issue order) and the compute warps finished reading this tile's S^T before P_ready.
          if (more) {
            const int s1 = (gi + 1) % NQS;
            if (!mbar_wait(&q_full[s1], ((gi + 1) / NQS) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after_sync();
            issue_s(gi + 1);
            umma_commit(s_full);
          }
          if (!mbar_wait(ds_ready, gi & 1, abort_flag)) { ok = false; break; }
          tc_fence_after_sync();
          {
            // dK += dS^T Q: A = dS^T from shared memory (K-major: 64-query chunks, 32 bytes per 16 queries),
            // B = Q MN-major.
            uint64_t a = ds_kmaj, qd = sdesc_add(q_mn, s * L::kTile);
            opaque(a, qd);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_ss(tmem + L::kColDK, sdesc_add(a, (kk / 4) * 16384 + (kk % 4) * 32), sdesc_add(qd, kk * 2048),
                      id_kv, (it > 0 || kk > 0));
          }
          umma_commit(&q_empty[s]);
          // dQ^T = K^T dS^T into RP (the compute warps have read this tile's dP^T): A = K MN-major (head dim
          // contiguous), B = dS^T MN-major (queries contiguous), 16 keys (2048 bytes) per instruction. (Issuing
          // it before dK, so that its read-out overlaps dK, measured no faster: the dQ warps' reductions then
          // meet the issue of dK.)
          {
            uint64_t a = k_mn, bd = ds_mn;
            opaque(a, bd);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_ss(tmem + L::kColP, sdesc_add(a, kk * 2048), sdesc_add(bd, kk * 2048), id_q, kk > 0);
          }
          umma_commit(dq_full);
          umma_commit(ds_empty);
          if (more) {
            // The dQ read-out is the one wait on this thread's critical path (the tensor core idles through it),
            // so it polls without suspending (the dQ warps and the compute warps have slack; measured faster in
            // paired runs, while spinning on the other waits of this thread was slower).
            if (!mbar_wait_spin(dq_empty, gi & 1, abort_flag)) { ok = false; break; }
            tc_fence_after_sync();
            issue_dp(gi + 1);
            umma_commit(dp_full);
          }
        }
        if (!ok) break;
        // The unit's products are complete: its dK/dV may be read out and K/V reloaded.
        umma_commit(dkv_done);
        g += n_it;
        ++w;
      }
      // Every product issued (also on an abort, mid-unit) must be complete before TMEM is released.
      umma_commit(mma_drain);
      int drain = 0;
      mbar_wait(mma_drain, 0, &drain);
    }
  } else if (warp < 8) {
    regs_inc<L::kRegsWork>();
    // ------------------------------------------------------------------ compute warps (thread = key row)
    const int half = warp / 4;     // query columns 64 * half .. +63 of each tile
    const uint32_t quarter = warp % 4;
    const int j = quarter * 32 + lane;  // key row within the tile = TMEM lane
    const int cb = 64 * half;
    const uint32_t lane_base = tmem + ((quarter * 32) << 16);
    bool ok = true;
    int g = 0, w = 0;  // global iteration, units with work
    for (int u = 0; ok && u < n_units; ++u) {
      const Unit U = unit_at(u);
      const int key0 = U.key0, i_begin = U.i_begin, n_q = U.n_q, n_it = U.n_it;
      const int key = key0 + j;
      for (int it = 0; it < n_it; ++it) {
        const int gi = g + it;
        const int s = gi % NQS;
        const int q0 = (i_begin + it % n_q) * BQ;
        const float* lse2 = reinterpret_cast<const float*>(smem_raw + L::kLOff + s * BQ * 4) + cb;
        const float* dvec = reinterpret_cast<const float*>(smem_raw + L::kDVecOff + s * BQ * 4) + cb;
        // This key's visible queries are [key - off - right, key - off + left]: columns (tile-relative) outside
        // [lo_c, hi_c] are masked; a tile every key of this CTA sees whole needs no element mask.
        const int lo_c = has_right ? key - off - right - q0 : -1;
        const int hi_c = has_left ? key - off + p.win_left - q0 : BQ;
        const bool need_mask =
            (has_right && key0 + 127 - off - right > q0) || (has_left && key0 - off + p.win_left < q0 + BQ - 1);
        // ---- P^T from S^T (64 columns of this warpgroup), kept in fp32 for dS^T; 16-bit P^T (times the keep
        // mask with dropout) back into TMEM over the first 32 of these columns. The dropout mask is generated
        // first, while S^T may still be in flight.
        uint64_t keep = 0;  // with dropout: bit c = query cb + c kept
        if constexpr (kDrop) {
          // Mask bytes of queries cb .. cb + 63 for this key: per 16 queries the four lanes of this key's 4-key
          // block each generate one 4x4 block, transpose its bytes (word = key) and exchange words, so that
          // kw[k] holds this key's bytes for queries cb + 16 g + 4 k .. + 3; thresholded into one bit per query.
          const uint32_t bhq = static_cast<uint32_t>(b * p.H + h_kv * p.group + it / n_q);
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            uint32_t kw[4];
            philox4x32_10(static_cast<uint32_t>((q0 + cb + 16 * g) >> 2) + (lane & 3u), static_cast<uint32_t>(key >> 2),
                          bhq, p.drop_off, p.drop_k0, p.drop_k1, kw);
            byte_transpose4(kw);
            quad_exchange(kw);
#pragma unroll
            for (int c = 0; c < 16; ++c)
              keep |= static_cast<uint64_t>(keep_byte(kw[c / 4], c % 4, p.drop_t)) << (16 * g + c);
          }
        }
        auto kept = [&](int c) { return ((keep >> c) & 1ull) != 0ull; };
        // (the empty asm statements make each loop extract its bits from `keep` instead of the compiler keeping
        // 64 separate flags alive across both phases)
        asm volatile("" : "+l"(keep));
        if (!mbar_wait(s_full, gi & 1, abort_flag)) { ok = false; break; }
        tc_fence_after_sync();
        float pv[64];
        tmem_ld_x64(lane_base + L::kColS + cb, reinterpret_cast<uint32_t*>(pv));
        {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            const float4 l4 = *reinterpret_cast<const float4*>(lse2 + c);
            float p0 = ex2_approx(fmaf(pv[c], p.scale_log2, -l4.x));
            float p1 = ex2_approx(fmaf(pv[c + 1], p.scale_log2, -l4.y));
            float p2 = ex2_approx(fmaf(pv[c + 2], p.scale_log2, -l4.z));
            float p3 = ex2_approx(fmaf(pv[c + 3], p.scale_log2, -l4.w));
            if (need_mask) {
              if (cb + c < lo_c || cb + c > hi_c) p0 = 0.f;
              if (cb + c + 1 < lo_c || cb + c + 1 > hi_c) p1 = 0.f;
              if (cb + c + 2 < lo_c || cb + c + 2 > hi_c) p2 = 0.f;
              if (cb + c + 3 < lo_c || cb + c + 3 > hi_c) p3 = 0.f;
            }
            pv[c] = p0;
            pv[c + 1] = p1;
            pv[c + 2] = p2;
            pv[c + 3] = p3;
            if constexpr (kDrop) {
              // dV takes the kept P (its 1/(1-t/256) is applied to dV at the end)
              pk[c / 2] = pack2<kBF16>(kept(c) ? p0 : 0.f, kept(c + 1) ? p1 : 0.f);
              pk[c / 2 + 1] = pack2<kBF16>(kept(c + 2) ? p2 : 0.f, kept(c + 3) ? p3 : 0.f);
            } else {
              pk[c / 2] = pack2<kBF16>(p0, p1);
              pk[c / 2 + 1] = pack2<kBF16>(p2, p3);
            }
          }
          tmem_st_x32(lane_base + L::kColS + cb, pk);
        }
        tmem_st_wait();
        tc_fence_before_sync();
        mbar_arrive(p_ready);
        // ---- dS^T = P^T (dP^T - D) (with dropout, dP reaching P is Z * (dO . v): 0 where dropped, scaled by
        // 1/(1-t/256) where kept), 16-bit, into this warpgroup's 64-query chunk of the dS^T buffer.
        if (!mbar_wait(dp_full, gi & 1, abort_flag)) { ok = false; break; }
        // The dS^T buffer is free once the previous tile's dK and dQ^T products have read it.
        if (gi >= 1 && !mbar_wait(ds_empty, (gi - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after_sync();
        // Row j of chunk `half` of the buffer: one 128-byte row, 16-byte units (8 queries) at the 128-byte-swizzle
        // positions; 32 queries (four units) at a time.
        uint8_t* ds_row = smem + L::kDSOff + half * 16384 + j * 128;
        asm volatile("" : "+l"(keep));
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 32) {
          float dp[32];
          tmem_ld_x32(lane_base + L::kColP + cb + c0, reinterpret_cast<uint32_t*>(dp));
          uint32_t dsk[16];
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            const float4 d4 = *reinterpret_cast<const float4*>(dvec + c0 + c);
            float g0 = dp[c], g1 = dp[c + 1], g2 = dp[c + 2], g3 = dp[c + 3];
            if constexpr (kDrop) {
              const float z = p.drop_scale;
              g0 = kept(c0 + c) ? g0 * z : 0.f;
              g1 = kept(c0 + c + 1) ? g1 * z : 0.f;
              g2 = kept(c0 + c + 2) ? g2 * z : 0.f;
              g3 = kept(c0 + c + 3) ? g3 * z : 0.f;
            }
            dsk[c / 2] = pack2<kBF16>(pv[c0 + c] * (g0 - d4.x), pv[c0 + c + 1] * (g1 - d4.y));
            dsk[c / 2 + 1] = pack2<kBF16>(pv[c0 + c + 2] * (g2 - d4.z), pv[c0 + c + 3] * (g3 - d4.w));
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int unit = c0 / 8 + u;
            *reinterpret_cast<uint4*>(ds_row + ((unit ^ (j & 7)) * 16)) =
                make_uint4(dsk[4 * u], dsk[4 * u + 1], dsk[4 * u + 2], dsk[4 * u + 3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        mbar_arrive(ds_ready);
      }
      // ---------------------------------------------------------------- epilogue: dV and dK rows
      if (ok && n_it > 0) ok = mbar_wait(dkv_done, w & 1, abort_flag);
      if (ok) {
        tc_fence_after_sync();
        // Each warp stages its 32 rows x 64 columns of dV, then dK, in its own 4 KB of the dS^T buffer (the rows
        // it writes dS^T to, free now that the unit's products are complete): written row by row (one row per
        // lane, 16-byte units XOR-swizzled by row so that the stores do not collide in banks), read back four
        // rows per instruction, so that each global store writes four whole 128-byte pieces of rows instead of
        // 32 scattered 16-byte ones (measured: the scattered stores made a unit's epilogue ~4 us longer).
        uint8_t* stage = smem + L::kDSOff + half * 16384 + quarter * 4096;
#pragma unroll
        for (int which = 0; which < 2; ++which) {
          const float mul = which == 0 ? (kDrop ? p.drop_scale : 1.f) : p.scale;
          const uint32_t col = (which == 0 ? L::kColDV : L::kColDK) + cb;
#pragma unroll
          for (int c0 = 0; c0 < 64; c0 += 32) {
            float v[32];
            if (n_it > 0) {
              tmem_ld_x32(lane_base + col + c0, reinterpret_cast<uint32_t*>(v));
            } else {
#pragma unroll
              for (int c = 0; c < 32; ++c) v[c] = 0.f;
            }
            uint32_t wd[16];
#pragma unroll
            for (int c = 0; c < 32; c += 2) wd[c / 2] = pack2<kBF16>(v[c] * mul, v[c + 1] * mul);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const int cc = c0 / 8 + q4;  // 16-byte unit of this row's 128 bytes
              *reinterpret_cast<uint4*>(stage + lane * 128 + ((cc ^ (lane & 7)) * 16)) =
                  make_uint4(wd[4 * q4], wd[4 * q4 + 1], wd[4 * q4 + 2], wd[4 * q4 + 3]);
            }
          }
          __syncwarp();
          uint16_t* dst = reinterpret_cast<uint16_t*>(which == 0 ? p.dv : p.dk);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = 4 * i + static_cast<int>(lane >> 3), cc = static_cast<int>(lane & 7);
            const uint4 val = *reinterpret_cast<const uint4*>(stage + r * 128 + ((cc ^ (r & 7)) * 16));
            const int key_r = key0 + static_cast<int>(quarter) * 32 + r;
            if (key_r < p.Sk)
              *reinterpret_cast<uint4*>(dst + ((static_cast<size_t>(b) * p.Sk + key_r) * p.Hkv + h_kv) * 128 + cb +
                                        cc * 8) = val;
          }
          __syncwarp();
        }
      }
      g += n_it;
      if (n_it > 0) ++w;
    }
  } else {
    regs_inc<L::kRegsWork>();
    // ------------------------------------------------------------------ dQ warps (lane = head-dim index)
    const uint32_t quarter = warp - 8;
    const int d = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((quarter * 32) << 16);
    bool ok = true;
    int g = 0;  // global iteration
    for (int u = 0; ok && u < n_units; ++u) {
      const Unit U = unit_at(u);
      for (int it = 0; it < U.n_it; ++it) {
        const int gi = g + it;
        const int h = h_kv * p.group + it / U.n_q;
        const int q0 = (U.i_begin + it % U.n_q) * BQ;
        if (!mbar_wait(dq_full, gi & 1, abort_flag)) { ok = false; break; }
        tc_fence_after_sync();
        float v[128];
        tmem_ld_x64_pair(lane_base + L::kColP, reinterpret_cast<uint32_t*>(v), lane_base + L::kColP + 64,
                         reinterpret_cast<uint32_t*>(v + 64));
        tc_fence_before_sync();
        mbar_arrive(dq_empty);
        // Four queries of this head-dim index per 16-byte reduction; a warp covers 512 contiguous bytes. The
        // reductions are paced (a short sleep after each): issued back to back they fill the memory-instruction
        // queue of every SM sub-partition, and the MMA thread's tcgen05 instructions, which wait in the same queue,
        // stall behind them (measured, alternating runs on one B200: main kernel 6.26 -> 5.64 ms at
        // 4x32x8192x128, within 4% of a timing copy with no reductions at all). A tile's 64 KB need only ~15 bytes
        // per cycle of the ~23 an SM sustains. The sleep is bounded from both sides (paired runs): at 20-30 ns
        // the queues fill again (+18% time), and the 32 sleeps must end well inside one tile's ~5000 cycles, or
        // the dQ warps become the bottleneck (75 ns: +40%); 50 ns keeps a 20% margin at the top SM clock.
        float* base = p.dq_acc + ((static_cast<size_t>(b) * p.H + h) * (p.Sq_pad / 4) + q0 / 4) * 512 + d * 4;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          red_add_v4(base + static_cast<size_t>(c) * 512, v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
          __nanosleep(50);
        }
      }
      g += U.n_it;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// dQ = dtype(scale * dQacc) for head dim 128, reading the query-quad layout [B, H, Sq_pad / 4, 128, 4]: a thread
// takes four head-dim indices of four queries (64 contiguous bytes) and writes four 8-byte pieces, one per query
// row, so that a warp reads 2 KB contiguously and writes four whole 256-byte rows.
template <bool kBF16>
__global__ void __launch_bounds__(256) fa_bwd_dq128_kernel(const BwdParams p) {
  const int quads = p.Sq_pad / 4;
  const long long n = (long long)p.B * p.H * quads * 32;
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < n; t += (long long)gridDim.x * blockDim.x) {
    const int dg = (int)(t % 32);
    const long long r = t / 32;
    const int qq = (int)(r % quads);
    const long long bhq = r / quads;
    const int h = (int)(bhq % p.H), b = (int)(bhq / p.H);
    const float4* src = reinterpret_cast<const float4*>(p.dq_acc) + r * 128 + dg * 4;
    const float4 a0 = src[0], a1 = src[1], a2 = src[2], a3 = src[3];  // head dims 4dg .. 4dg+3, queries 4qq ..
    const float sc = p.scale;
    const float x[4][4] = {{a0.x, a1.x, a2.x, a3.x}, {a0.y, a1.y, a2.y, a3.y}, {a0.z, a1.z, a2.z, a3.z},
                           {a0.w, a1.w, a2.w, a3.w}};
#pragma unroll
    for (int rq = 0; rq < 4; ++rq) {
      const int i = qq * 4 + rq;
      if (i >= p.Sq) break;
      uint2 w;
      w.x = pack2<kBF16>(x[rq][0] * sc, x[rq][1] * sc);
      w.y = pack2<kBF16>(x[rq][2] * sc, x[rq][3] * sc);
      *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(p.dq) + ((static_cast<size_t>(b) * p.Sq + i) * p.H + h) * 128 +
                                dg * 4) = w;
    }
  }
}

}  // namespace fa
