// attn_kernel.cuh -- warp-specialised FMHA forward for sm_100a.
//
// Computes O = softmax(scale * Q K^T) V on dequantized operands with an
// online-softmax pass over 128-key tiles ("FlashInfer FP8/BF16 mixed-precision
// attention for Blackwell", introduction and section 1: QK (BMM1) -> softmax ->
// PV (BMM2); "FlashInfer DiT optimization: SageAttention and Int8/FP8
// mixed-precision kernels", section 2: Q/K/P/V scale factors applied after the
// 8-bit BMMs).
//
// One CTA owns two 128-row query tiles X = 0, 1 that share every K/V tile
// (either two consecutive query blocks of one head, or the same query block
// of two query heads that read the same KV head; for decode, GQA-packed tiles
// of one KV head's query heads). 384 threads, one CTA/SM:
//   warp  0     tensor-core issue (warp-uniform, one elected lane issues)
//   warp  1     TMA producer (warp-uniform; one tile's copies from several lanes)
//   warps 2-3   idle (warp 2 picks decode splits' KV tiles in the prologue);
//               warpgroup 0 hands its registers to the softmax with setmaxnreg
//   warps 4-7   softmax for tile 0 (TMEM lanes 0-127: one query row per thread)
//   warps 8-11  softmax for tile 1
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D).
// BF16 P is written over the first columns of its S tile and the PV product
// reads it from TMEM; the issue order puts S_X(j+1) after PV_X(j), so the
// arrival of S_X(j+1) proves PV_X(j) finished and the softmax rescales O itself
// (only when the running row max grows by more than 2^tau, the "lazy
// correction" of the Blackwell page, section 3) before releasing P_X(j+1).
// E4M3 P goes to shared memory instead (the Blackwell page, section 1), so a
// tile's S columns are free once the softmax has loaded them: QK^T of the next
// KV tile overlaps the softmax, and the two softmax warpgroups take turns in
// their exp2 phases.
// The epilogue scales O by 1/l (and the V / P scale factors), converts to BF16
// (64-column halves) or E4M3 (O / sf_o, one 128-byte row per query row), stages
// the result in the dead Q buffer and writes it with TMA stores ("FlashInfer
// DeepSeek-V4 sparse-MLA: Cake backend", section 1: output through a TMA
// descriptor passed as a grid constant).
//
// Every wait is bounded: on expiry the thread sets the device error word and a
// CTA-wide abort flag; all roles then fall through to a teardown that drains
// in-flight TMA loads and MMAs before TMEM is freed. Nothing traps.
#pragma once

#include "fmha_internal.h"
#include "ptx_sm100.cuh"

#include <type_traits>

namespace fmha {

// D: head dim of Q and K; DV: head dim of V and O (192 / 128 for a wide QK).
template <int D_, int QK_, int PV_, bool PAGED_, bool P2_ = false, bool PACKED_ = false, bool O8_ = false,
          int DV_ = D_>
struct AttnCfg {
  static constexpr int D = D_, DV = DV_, QK = QK_, PV = PV_;
  static constexpr bool PAGED = PAGED_;
  // GQA-packed query tiles and split-KV ranges (decode shapes).
  static constexpr bool PACKED = PACKED_;
  static constexpr bool P2 = P2_;  // E4M3 P split into two terms (hi + lo), each with its own PV product
  static_assert(!P2 || PV == PV_E4M3, "two-term P needs an E4M3 V");
  // E4M3 output: O / sf_o rounded to E4M3 (one 128-byte row per query row).
  static constexpr bool O8 = O8_;
  static_assert(!O8 || (DV == 128 && !PACKED), "E4M3 O is built for 128-wide O tiles");
  static_assert(DV == 64 || DV == 128, "V / O head dim 64 or 128");
  static constexpr int BM = 128, BN = 128;
  static constexpr int QK_ELEM = QK == QK_BF16 ? 2 : 1;
  static constexpr int V_ELEM = PV == PV_BF16 ? 2 : 1;
  static constexpr int QK_ROW_BYTES = D * QK_ELEM;
  // 128-byte swizzle columns along D. A 192-byte E4M3 row takes two: the copy
  // of the second reads 64 bytes past the row's end, which TMA fills with
  // zeros (they count in the transaction bytes; no MMA step reads them).
  static constexpr int QK_CHUNKS = (QK_ROW_BYTES + 127) / 128;
  static constexpr int QK_CHUNK_ELEMS = 128 / QK_ELEM;
  static constexpr int V_CHUNKS = DV * V_ELEM / 128;
  static constexpr int V_CHUNK_ELEMS = 128 / V_ELEM;
  static_assert(QK_ROW_BYTES % 64 == 0 && (DV * V_ELEM) % 128 == 0, "rows must be whole swizzle atoms");
  static constexpr int CHUNK_BYTES = 128 * 128;  // one 128-row x 128-byte swizzled column block
  static constexpr int Q_TILE = BM * QK_CHUNKS * 128;
  static constexpr int K_TILE = BN * QK_CHUNKS * 128;
  static constexpr int V_TILE = BN * DV * V_ELEM;
  static constexpr int SLOT = K_TILE > V_TILE ? K_TILE : V_TILE;
  // E4M3 P is staged in shared memory (one 128 x 128 byte tile per query tile
  // and term) so that a tile's S buffer in TMEM is free as soon as the softmax
  // has loaded it: QK^T of the next KV tile then overlaps this tile's exp2
  // ("FlashInfer FP8/BF16 mixed-precision attention for Blackwell", section 1).
  // BF16 P stays in TMEM (staging it would leave too little room for K/V).
  static constexpr bool PSMEM = PV == PV_E4M3;
  static constexpr bool TURNS = PSMEM;  // exp-phase turn-taking between the softmax warpgroups
  static constexpr int P_TILE = BM * BN;  // bytes per E4M3 P tile
  // Query tiles per CTA (1 when two 48 KB BF16 Q tiles would starve the K/V ring).
  static constexpr int NQ = query_tiles_per_cta(QK, D);
  static_assert(NQ == 2 || !PACKED, "decode tiles come in pairs");
  // One query tile: the two softmax warpgroups take alternate kept KV tiles of
  // it (an intra-CTA split of the keys), each with its own S, P and O, and the
  // epilogue merges the two partial results. K and V then have rings of their
  // own (2 slots each: a 48 KB K slot and a 32 KB V slot are not interchangeable).
  static constexpr bool SPLIT = NQ == 1;
  static_assert(!SPLIT || (!O8 && !P2), "split tiles: BF16 O, one-term P");
  static constexpr int P_BYTES = PSMEM ? 2 * P_TILE * (P2 ? 2 : 1) : 0;
  static constexpr int MISC_BYTES = 2048;
  static constexpr int SMEM_CAP = 232448;  // 227 KB opt-in maximum per CTA
  static constexpr int STAGES_FIT = (SMEM_CAP - 1024 - MISC_BYTES - NQ * Q_TILE - P_BYTES) / SLOT;
  static constexpr int STAGES = STAGES_FIT > 6 ? 6 : STAGES_FIT;
  static_assert(SPLIT || STAGES >= 3, "the K/V ring needs at least three slots");
  // Split rings: two K slots, and as many V slots (up to 4) as the rest holds.
  static constexpr int K_STAGES = 2;
  static constexpr int V_FIT = (SMEM_CAP - 1024 - MISC_BYTES - NQ * Q_TILE - P_BYTES - K_STAGES * K_TILE) / V_TILE;
  static constexpr int V_STAGES = V_FIT > 4 ? 4 : V_FIT;
  static_assert(!SPLIT || V_STAGES >= 2, "the V ring needs two slots");
  static constexpr int RING_BYTES = SPLIT ? K_STAGES * K_TILE + V_STAGES * V_TILE : STAGES * SLOT;
  static constexpr int SMEM_BYTES = 1024 + NQ * Q_TILE + P_BYTES + RING_BYTES + MISC_BYTES;
  static_assert(SMEM_BYTES <= SMEM_CAP, "shared memory");
  static constexpr int QK_STEPS = QK_ROW_BYTES / 32;  // one MMA covers 32 bytes of K (16 bf16 / 32 8-bit)
  static constexpr int PV_K = PV == PV_BF16 ? 16 : 32;
  static constexpr int PV_STEPS = BN / PV_K;
  static constexpr int O_STAGE_BUFS = Q_TILE / CHUNK_BYTES;  // 16 KB staging buffers inside a Q buffer
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t IDESC_QK = QK == QK_BF16   ? ptx::make_idesc(1, 1, 1, 0, 0, BN, BM)
                                       : QK == QK_E4M3 ? ptx::make_idesc(1, 0, 0, 0, 0, BN, BM)
                                                       : ptx::make_idesc(2, 1, 1, 0, 0, BN, BM);
  static constexpr uint32_t IDESC_PV =
      PV == PV_BF16 ? ptx::make_idesc(1, 1, 1, 0, 1, DV, BM) : ptx::make_idesc(1, 0, 0, 0, 1, DV, BM);
  static constexpr int THREADS = 384;
  // Warp roles: warpgroup 0 = control (MMA issue, TMA loads, two idle warps),
  // warpgroups 1 and 2 = softmax of query tiles 0 and 1 (one thread per row).
  // The control warps come first: the issue scheduler favours older warps, and
  // the MMA warp's short serial steps sit on the critical path of both softmax
  // pipelines.
  static constexpr int MMA_WARP = 0, LOAD_WARP = 1, SOFTMAX_WARP0 = 4;
  // setmaxnreg split of the launch's registers (384 threads x 168):
  // 2 * 128 * 216 + 128 * 72.
  static constexpr uint32_t SOFTMAX_REGS = 216, CONTROL_REGS = 72;
  static_assert(2 * 128 * SOFTMAX_REGS + 128 * CONTROL_REGS <= THREADS * 168, "register split exceeds launch");
};

struct alignas(8) AttnMisc {
  uint64_t q_full;
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full;
  uint64_t drain;
  uint64_t s_free[2];   // shared-memory P: the softmax has loaded S, its TMEM may be overwritten
  uint64_t pv_done[2];  // shared-memory P: a PV product finished (O current, P buffer free)
  uint64_t exp_done[2];  // softmax warpgroup x finished the exponentials of its current tile
  uint64_t kv_full[8];
  uint64_t kv_empty[8];
  uint32_t tmem_base;
  volatile uint32_t abort;
  float sf_v[128];
  // The KV tiles each query tile processes, as a bit set over KV tiles (at
  // most 1024), for packed (decode) CTAs and for every launch with a block
  // mask: built once in the prologue, so no role reads the mask per tile.
  uint32_t keep_bits[2][32];
  int32_t range[2][2];  // packed: [first, last + 1) of each query tile's kept tiles
  int32_t same_kept;    // masked: both query tiles keep the same KV tiles (count), else 0;
                        // split tiles: the kept tiles each warpgroup has at least
};

static_assert(sizeof(AttnMisc) <= 2048, "AttnMisc must fit the 2 KB misc area");

struct TileInfo {
  int h;      // query head (packed: first head of the KV head's group)
  int q0;     // first row (packed: first packed row, = token * group + head in group)
  int qblk;   // 128-row block index
  int tok0;   // first query token
  int mrow;   // block-mask row (128-token query block)
  int u0;     // KV tiles [u0, n_kv) not excluded by causality, length or split
  int n_kv;
  int x;      // query tile slot in the CTA (0 or 1)
  int part;   // packed, several partials: index of this tile's partial output
  bool valid;
};

// Suspend-time hint of one barrier probe, in ns.
constexpr uint32_t kWaitSleepNs = 1000;

// Bounded mbarrier wait. Returns false on timeout (recorded) or CTA abort.
struct Waiter {
  volatile uint32_t* abort_flag;
  uint32_t* err;
  uint64_t budget;
  __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity) const {
    // First a non-blocking test: try_wait may itself suspend the thread for a
    // hardware-chosen time, which would let a short limit never run out.
    if (ptx::mbar_test_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
      // The limit is checked before every sleeping probe, so a limit shorter
      // than one probe still gives up after the first unsatisfied probe.
      if (static_cast<uint64_t>(clock64() - t0) > budget) {
        *abort_flag = 1u;
        record_timeout(bar, parity);
        return false;
      }
      // Sleep in the barrier (woken when the phase completes) rather than spin:
      // a spinning warp takes issue slots from the warps sharing its scheduler.
      if (ptx::mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
      if (*abort_flag) return false;
    }
  }
  // Sets the timeout bit and, for the first timeout only, the site bits.
  __device__ __forceinline__ void record_timeout(uint32_t bar, uint32_t parity) const {
    const uint32_t site = ((bar & 0xfffu) | ((parity & 1u) << 12) | (((threadIdx.x >> 5) + 1u) << 16))
                          << kErrSiteShift;
    uint32_t old = atomicOr(err, kErrTimeout);
    for (int tries = 0; tries < 8 && (old >> kErrSiteShift) == 0u; ++tries) {
      const uint32_t seen = atomicCAS(err, old | kErrTimeout, old | kErrTimeout | site);
      if (seen == (old | kErrTimeout)) break;
      old = seen;
    }
  }
  // Teardown wait: ignores the abort flag (used to drain in-flight async work).
  // Its limit never drops below ~1 s, whatever the wait limit is set to: a copy
  // or MMA already issued always completes, and shared memory / TMEM must not
  // be released under it.
  __device__ __forceinline__ bool drain(uint32_t bar, uint32_t parity) const {
    const uint64_t limit = budget > (1ull << 31) ? budget : (1ull << 31);
    const long long t0 = clock64();
    while (!ptx::mbar_try_wait(bar, parity)) {
      if (static_cast<uint64_t>(clock64() - t0) > limit) {
        record_timeout(bar, parity);
        return false;
      }
    }
    return true;
  }
};

// Tile info and waiters are passed by value everywhere: a runtime-indexed
// array or a by-reference argument would live in local memory, and with the
// shared-memory carve-out near its maximum every such load goes to L2.
// Whether the CTA's KV tiles are listed in the keep-bit set (packed CTAs: the
// split's tiles; masked launches: the block mask's kept tiles).
template <class C>
__device__ __forceinline__ bool uses_keep_bits(const AttnParams& p) {
  return C::PACKED || C::SPLIT || p.mask != nullptr;
}

template <class C>
__device__ __forceinline__ bool keep_tile(const AttnParams& p, const TileInfo t, int u, const AttnMisc* misc) {
  if (u < t.u0 || u >= t.n_kv) return false;
  if (!uses_keep_bits<C>(p)) return true;
  return (misc->keep_bits[t.x][u >> 5] >> (u & 31)) & 1u;
}

// First KV tile at or after `from` (and below n) kept by the query tiles whose
// bits `sel` selects (1: tile 0, 2: tile 1, 3: either); n when none.
template <class C>
__device__ __forceinline__ int next_kept_tile(const AttnParams& p, const AttnMisc* misc, int sel, int from, int n) {
  if (from >= n) return n;
  if (!uses_keep_bits<C>(p)) return from;
  for (int wd = from >> 5; (wd << 5) < n; ++wd) {
    uint32_t bits = ((sel & 1) ? misc->keep_bits[0][wd] : 0u) | ((sel & 2) ? misc->keep_bits[1][wd] : 0u);
    if (wd == (from >> 5)) bits &= ~0u << (from & 31);
    if (bits) return min(n, (wd << 5) + __ffs(bits) - 1);
  }
  return n;
}

__device__ __forceinline__ float sf_lookup(const float* sf, int kind, int64_t bh, int nblk, int idx_in_seq,
                                           int rpb) {
  switch (kind) {
    case FMHA_SF_PER_TENSOR: return sf[0];
    case FMHA_SF_PER_HEAD: return sf[bh];
    case FMHA_SF_PER_TOKEN_BLOCK: return sf[bh * nblk + idx_in_seq / rpb];
    default: return 1.f;
  }
}

// ------------------------------------------------------------ TMA producer --
template <class C>
// TMA producer, run by the whole warp: the schedule (kept tiles, slots,
// phases) is warp-uniform; lane 0 posts each slot's expected bytes, then the
// copies of one tile (chunks x pages) are issued from different lanes at once,
// and for paged K/V each lane reads the page-table entry of its page.
__device__ void attn_load_role(const AttnParams& p, const TileInfo t0, const TileInfo t1, int b, int hkv,
                               uint8_t* sQ0, uint8_t* sQ1, uint8_t* sSlots, AttnMisc* misc, const CUtensorMap* tmQ,
                               const CUtensorMap* tmK, const CUtensorMap* tmV, const Waiter w) {
  using namespace ptx;
  constexpr uint32_t FULL = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  const TileInfo t[2] = {t0, t1};  // indexed only with unrolled constants below
  uint8_t* const sQ[2] = {sQ0, sQ1};
  const uint32_t q_full = smem_addr(&misc->q_full);
  if (lane == 0) {
    uint32_t qbytes = 0;
#pragma unroll
    for (int x = 0; x < 2; ++x) qbytes += t[x].valid ? C::Q_TILE : 0;
    mbar_arrive_expect_tx(q_full, qbytes);
  }
  __syncwarp();
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    if (!t[x].valid) continue;
#pragma unroll
    for (int c = 0; c < C::QK_CHUNKS; ++c) {
      if (lane != x * C::QK_CHUNKS + c) continue;
      if constexpr (C::PACKED)  // box: all heads of the group x 128 / group tokens
        tma_load_5d(smem_addr(sQ[x]) + c * C::CHUNK_BYTES, tmQ, q_full, c * C::QK_CHUNK_ELEMS, 0, hkv, t[x].tok0,
                    b);
      else
        tma_load_4d(smem_addr(sQ[x]) + c * C::CHUNK_BYTES, tmQ, q_full, c * C::QK_CHUNK_ELEMS, t[x].h, t[x].q0, b);
    }
  }
  const uint64_t pol = policy_evict_last();  // K/V tiles are re-read by every CTA of this head
  uint32_t issued = 0u, issued_phase = 0u;  // per slot: a load was issued / parity of its last phase
  int slot_it = 0;
  const int n_u = max(t0.n_kv, t1.n_kv);
  bool ok = true;
  // Next KV tile at or after `from` that either query tile keeps.
  auto next_kept = [&](int from) { return next_kept_tile<C>(p, misc, 3, from, n_u); };
  // Paged K/V: lane l reads the page-table entry of page l of a tile (BN /
  // page_size <= 8 pages) once for its K and V copies, one kept tile ahead.
  const int per = C::PAGED ? C::BN / p.page_size : 1;
  auto lookup = [&](int v) {
    int e = -1;
    const int lp = v * per + lane;  // logical page of this sequence
    if (C::PAGED && lane < per && lp * p.page_size < p.Skv)
      e = __ldg(p.page_table + static_cast<int64_t>(b) * p.max_pages_per_seq + lp);
    return e;
  };
  // One kept tile u: lane l issues copy l (page l / chunks, chunk l % chunks)
  // of K, then of V, using the page entry read one tile earlier (`cur`).
  auto step = [&](int& u, int& cur, int& nxt) {
    const int nu = next_kept(u + 1);
    int page = 0;
    if constexpr (C::PAGED) {
      if (nu < n_u) nxt = lookup(nu);
      const int lp = u * per + lane;
      const bool in_seq = lane < per && lp * p.page_size < p.Skv;
      if (in_seq && (cur < 0 || cur >= p.num_pages)) atomicOr(p.err, kErrPageIndex);
      page = (in_seq && cur >= 0 && cur < p.num_pages) ? cur : p.num_pages;  // out of range: TMA reads zeros
    }
    for (int kv = 0; kv < 2; ++kv) {  // K then V
      const int s = slot_it % C::STAGES;
      const uint32_t ph = (slot_it / C::STAGES) & 1;
      ++slot_it;
      if (!(ok = __all_sync(FULL, w.wait(smem_addr(&misc->kv_empty[s]), ph ^ 1)))) break;
      const uint32_t full = smem_addr(&misc->kv_full[s]);
      const int chunks = kv == 0 ? C::QK_CHUNKS : C::V_CHUNKS;
      const int chunk_elems = kv == 0 ? C::QK_CHUNK_ELEMS : C::V_CHUNK_ELEMS;
      const CUtensorMap* tm = kv == 0 ? tmK : tmV;
      const uint32_t dst = smem_addr(sSlots + s * C::SLOT);
      if (lane == 0) mbar_arrive_expect_tx(full, kv == 0 ? C::K_TILE : C::V_TILE);
      __syncwarp();
      issued |= 1u << s;
      issued_phase = (issued_phase & ~(1u << s)) | (ph << s);
      if constexpr (!C::PAGED) {
        if (lane < chunks)
          tma_load_4d_hint(dst + lane * C::CHUNK_BYTES, tm, full, lane * chunk_elems, hkv, u * C::BN, b, pol);
      } else {
        const int pp = lane / chunks, c = lane - pp * chunks;
        const int pg = __shfl_sync(FULL, page, pp & 31);
        if (pp < per)
          tma_load_4d_hint(dst + c * C::CHUNK_BYTES + pp * p.page_size * 128, tm, full, c * chunk_elems, hkv, 0, pg,
                           pol);
      }
    }
    u = nu;
  };
  int u = next_kept(min(t0.u0, t1.u0));
  int pg_a = -1, pg_b = -1;
  if constexpr (C::PAGED) {
    if (u < n_u) pg_a = lookup(u);
  }
  while (u < n_u && ok) {  // two alternating page registers: no copy waits for a pending lookup
    step(u, pg_a, pg_b);
    if (u >= n_u || !ok) break;
    step(u, pg_b, pg_a);
  }
  // Every issued copy lands before shared memory goes away. Without an abort
  // the consumers have already seen these phases complete (no waiting); after
  // an abort, set by any role at any time, copies may still be in flight.
  if (lane == 0) {
    w.drain(q_full, 0);
    for (int s = 0; s < C::STAGES; ++s)
      if (issued & (1u << s)) w.drain(smem_addr(&misc->kv_full[s]), (issued_phase >> s) & 1u);
  }
  __syncwarp();
}

// TMA producers for split tiles (one query tile, two softmax warpgroups taking
// alternate kept KV tiles): one warp loads Q and then the kept K tiles into
// the K ring (kv = 0), another the kept V tiles into the V ring (kv = 1), so
// neither ring's free slots wait on the other's. Barriers: kv_full/kv_empty
// [0, K_STAGES) for K, [K_STAGES, K_STAGES + V_STAGES) for V.
template <class C>
__device__ void attn_load_role_split(const AttnParams& p, const TileInfo t0, int b, int hkv, int kv_sel,
                                     uint8_t* sQ, uint8_t* sK, uint8_t* sV, AttnMisc* misc,
                                     const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                     const Waiter w) {
  using namespace ptx;
  constexpr uint32_t FULL = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  const uint32_t q_full = smem_addr(&misc->q_full);
  if (kv_sel == 0) {
    if (lane == 0) mbar_arrive_expect_tx(q_full, C::Q_TILE);
    __syncwarp();
    if (lane < C::QK_CHUNKS)
      tma_load_4d(smem_addr(sQ) + lane * C::CHUNK_BYTES, tmQ, q_full, lane * C::QK_CHUNK_ELEMS, t0.h, t0.q0, b);
  }
  const uint64_t pol = policy_evict_last();  // K/V tiles are re-read by every CTA of this head
  const int ring = kv_sel ? C::K_STAGES : 0, stages = kv_sel ? C::V_STAGES : C::K_STAGES;
  const int chunks = kv_sel == 0 ? C::QK_CHUNKS : C::V_CHUNKS;
  const int chunk_elems = kv_sel == 0 ? C::QK_CHUNK_ELEMS : C::V_CHUNK_ELEMS;
  const uint32_t tile_bytes = kv_sel == 0 ? C::K_TILE : C::V_TILE;
  const CUtensorMap* tm = kv_sel == 0 ? tmK : tmV;
  const uint32_t ring_base = smem_addr(kv_sel == 0 ? sK : sV);
  int pos = 0;  // tiles issued into this ring
  bool ok = true;
  const int n = t0.n_kv;
  const int per = C::PAGED ? C::BN / p.page_size : 1;
  // One tile u into the ring: lane l issues copy l (page l / chunks, chunk
  // l % chunks), the page entry read here.
  auto load = [&](int u) {
    const int s = pos % stages;
    const uint32_t ph = (pos / stages) & 1;
    if (!(ok = __all_sync(FULL, w.wait(smem_addr(&misc->kv_empty[ring + s]), ph ^ 1)))) return;
    ++pos;
    const uint32_t full = smem_addr(&misc->kv_full[ring + s]);
    const uint32_t dst = ring_base + s * tile_bytes;
    if (lane == 0) mbar_arrive_expect_tx(full, tile_bytes);
    __syncwarp();
    if constexpr (!C::PAGED) {
      if (lane < chunks)
        tma_load_4d_hint(dst + lane * C::CHUNK_BYTES, tm, full, lane * chunk_elems, hkv, u * C::BN, b, pol);
    } else {
      const int pp = lane / chunks, c = lane - pp * chunks;
      const int lp = u * per + pp;  // logical page of this sequence
      int pg = p.num_pages;         // out of range: TMA reads zeros
      if (pp < per && lp * p.page_size < p.Skv) {
        const int e = __ldg(p.page_table + static_cast<int64_t>(b) * p.max_pages_per_seq + lp);
        if (e < 0 || e >= p.num_pages) atomicOr(p.err, kErrPageIndex);
        else pg = e;
      }
      if (pp < per)
        tma_load_4d_hint(dst + c * C::CHUNK_BYTES + pp * p.page_size * 128, tm, full, c * chunk_elems, hkv, 0, pg,
                         pol);
    }
  };
  for (int u = next_kept_tile<C>(p, misc, 3, t0.u0, n); u < n && ok; u = next_kept_tile<C>(p, misc, 3, u + 1, n))
    load(u);
  // Every issued copy lands before shared memory goes away (see attn_load_role):
  // the last `stages` tiles issued, one per slot.
  if (lane == 0) {
    if (kv_sel == 0) w.drain(q_full, 0);
    for (int k = pos > stages ? pos - stages : 0; k < pos; ++k)
      w.drain(smem_addr(&misc->kv_full[ring + k % stages]), (k / stages) & 1u);
  }
  __syncwarp();
}

// ------------------------------------------------------- tensor-core issue --
// Descriptor words: lo = start address >> 4 | leading byte offset >> 4 << 16,
// hi = stride byte offset >> 4 | version 1 (bit 46) | swizzle (bits 61-63).
__device__ __forceinline__ uint32_t desc_lo(uint32_t addr, uint32_t lbo) {
  return ((addr & 0x3FFFFu) >> 4) | ((lbo >> 4) << 16);
}
__device__ __forceinline__ uint32_t desc_hi(uint32_t sbo, uint32_t swizzle) {
  return (sbo >> 4) | (1u << 14) | (swizzle << 29);
}

// S = Q K^T: QK_STEPS MMAs of K = 32 bytes; the K-step advances the start
// address by 32 bytes inside a 128-byte swizzle row, then jumps to the next
// 16 KB column block.
template <class C>
__device__ __forceinline__ void issue_qk(uint32_t tmem_d, uint32_t q_lo, uint32_t k_lo, uint32_t hi) {
#pragma unroll
  for (int s = 0; s < C::QK_STEPS; ++s) {
    const uint32_t off = ((s / 4) * C::CHUNK_BYTES + (s % 4) * 32) >> 4;
    if constexpr (C::QK == QK_BF16) {
      if (s == 0) ptx::mma_ss_f16_lean<false>(tmem_d, q_lo + off, hi, k_lo + off, hi, C::IDESC_QK);
      else ptx::mma_ss_f16_lean<true>(tmem_d, q_lo + off, hi, k_lo + off, hi, C::IDESC_QK);
    } else if constexpr (C::QK == QK_E4M3) {
      if (s == 0) ptx::mma_ss_f8_lean<false>(tmem_d, q_lo + off, hi, k_lo + off, hi, C::IDESC_QK);
      else ptx::mma_ss_f8_lean<true>(tmem_d, q_lo + off, hi, k_lo + off, hi, C::IDESC_QK);
    } else {
      if (s == 0) ptx::mma_ss_i8_lean<false>(tmem_d, q_lo + off, hi, k_lo + off, hi, C::IDESC_QK);
      else ptx::mma_ss_i8_lean<true>(tmem_d, q_lo + off, hi, k_lo + off, hi, C::IDESC_QK);
    }
  }
}

// O += P V: P (A operand) from TMEM, V MN-major in shared memory (d contiguous):
// K-step s starts PV_K rows down; the 64- or 128-wide d column blocks are
// CHUNK_BYTES apart (leading byte offset), 8-row groups 1 KB apart.
template <class C>
__device__ __forceinline__ void issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint32_t v_lo, uint32_t hi,
                                         uint32_t accumulate) {
#pragma unroll
  for (int s = 0; s < C::PV_STEPS; ++s) {
    const uint32_t off = (s * C::PV_K * 128) >> 4;
    const uint32_t acc = s > 0 ? 1u : accumulate;
    if constexpr (C::PV == PV_BF16)
      ptx::mma_ts_f16_lean(tmem_o, tmem_p + s * 8, v_lo + off, hi, C::IDESC_PV, acc);
    else
      ptx::mma_ts_f8_lean(tmem_o, tmem_p + s * 8, v_lo + off, hi, C::IDESC_PV, acc);
  }
}

// MMA issue (TMEM P). The whole warp walks the schedule -- waits, slot and
// phase bookkeeping, descriptor words -- in warp-uniform control flow, and one
// elected lane issues the MMAs and commits, so the address arithmetic stays
// off the issuing lane's critical path.
template <class C>
__device__ void attn_mma_role(const AttnParams& p, const TileInfo t0, const TileInfo t1, int b, int hkv, uint8_t* sQ0,
                              uint8_t* sQ1, uint8_t* sSlots, AttnMisc* misc, uint32_t tmem, const Waiter w) {
  using namespace ptx;
  constexpr uint32_t FULL = 0xffffffffu;
  const bool leader = elect_one();
  const uint32_t s_col[2] = {0u, 128u};
  // Descriptor words, computed once: K-major Q/K (leading offset unused, 16),
  // MN-major V (leading offset = distance between d column blocks).
  const uint32_t hi = desc_hi(1024, 2);
  const uint32_t q_lo0 = desc_lo(smem_addr(sQ0), 16), q_lo1 = desc_lo(smem_addr(sQ1), 16);
  const uint32_t k_lo0 = desc_lo(smem_addr(sSlots), 16);
  const uint32_t v_lo0 = desc_lo(smem_addr(sSlots), C::CHUNK_BYTES);
  const uint32_t o_col[2] = {256u, 256u + C::DV};
  int pend[2] = {-1, -1};
  int pv_cnt[2] = {0, 0};
  int prev_v = -1;
  int slot_it = 0;
  const int n_u = max(t0.n_kv, t1.n_kv);
  bool ok = __all_sync(FULL, w.wait(smem_addr(&misc->q_full), 0));
  tc_fence_after();
  for (int u = next_kept_tile<C>(p, misc, 3, min(t0.u0, t1.u0), n_u); u < n_u && ok;
       u = next_kept_tile<C>(p, misc, 3, u + 1, n_u)) {
    const bool kx[2] = {keep_tile<C>(p, t0, u, misc), keep_tile<C>(p, t1, u, misc)};
    const int ks = slot_it % C::STAGES;
    const uint32_t kph = (slot_it / C::STAGES) & 1;
    ++slot_it;
    const int vs = slot_it % C::STAGES;
    const uint32_t vph = (slot_it / C::STAGES) & 1;
    ++slot_it;
    bool k_ready = false;
    // Pass 1, query tiles that keep u: their pending PV (S_x(u) overwrites P_x
    // in TMEM), then S_x(u). Pass 2, tiles that skip u: their pending PV, after
    // the S MMAs above, so a tile whose softmax is still running does not hold
    // back the other tile's S.
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
      for (int x = 0; x < 2 && ok; ++x) {
        if (kx[x] != (pass == 0)) continue;
        if (pend[x] >= 0) {
          if (!(ok = __all_sync(FULL, w.wait(smem_addr(&misc->p_full[x]), pv_cnt[x] & 1)))) break;
          tc_fence_after();
          if (leader) {
            issue_pv<C>(tmem + o_col[x], tmem + s_col[x], v_lo0 + pend[x] * (C::SLOT >> 4), hi, pv_cnt[x] > 0);
            if constexpr (C::P2)  // the low E4M3 term of P
              issue_pv<C>(tmem + o_col[x], tmem + s_col[x] + 32, v_lo0 + pend[x] * (C::SLOT >> 4), hi, 1u);
          }
          __syncwarp();
          ++pv_cnt[x];
          pend[x] = -1;
        }
        if (kx[x]) {
          if (!k_ready) {
            if (!(ok = __all_sync(FULL, w.wait(smem_addr(&misc->kv_full[ks]), kph)))) break;
            tc_fence_after();
            k_ready = true;
          }
          if (leader) {
            issue_qk<C>(tmem + s_col[x], x ? q_lo1 : q_lo0, k_lo0 + ks * (C::SLOT >> 4), hi);
            tc_commit(smem_addr(&misc->s_full[x]));
          }
          __syncwarp();
        }
      }
    }
    if (!ok) break;
    if (leader) {
      tc_commit(smem_addr(&misc->kv_empty[ks]));                     // K_u free once the S MMAs finish
      if (prev_v >= 0) tc_commit(smem_addr(&misc->kv_empty[prev_v]));  // previous V: its PVs are issued
    }
    __syncwarp();
    if (!(ok = __all_sync(FULL, w.wait(smem_addr(&misc->kv_full[vs]), vph)))) break;
    tc_fence_after();
    pend[0] = kx[0] ? vs : -1;
    pend[1] = kx[1] ? vs : -1;
    prev_v = vs;
  }
#pragma unroll
  for (int x = 0; x < 2 && ok; ++x) {
    if (pend[x] < 0) continue;
    if (!(ok = __all_sync(FULL, w.wait(smem_addr(&misc->p_full[x]), pv_cnt[x] & 1)))) break;
    tc_fence_after();
    if (leader) {
      issue_pv<C>(tmem + o_col[x], tmem + s_col[x], v_lo0 + pend[x] * (C::SLOT >> 4), hi, pv_cnt[x] > 0);
      if constexpr (C::P2)
        issue_pv<C>(tmem + o_col[x], tmem + s_col[x] + 32, v_lo0 + pend[x] * (C::SLOT >> 4), hi, 1u);
    }
    __syncwarp();
  }
  // Drain: arrives when every MMA issued above has completed.
  if (leader) {
    if (ok) tc_commit(smem_addr(&misc->o_full));
    tc_commit(smem_addr(&misc->drain));
  }
  __syncwarp();
  w.drain(smem_addr(&misc->drain), 0);
}

// MMA issue for split tiles with P in TMEM (BF16 P). Kept tiles alternate
// between the softmax warpgroups (tile x = the keep-bit owner of u). Per kept
// tile u of warpgroup x: its pending PV_x (P_x lives over S_x in TMEM, so it
// must precede S_x(u)), then S_x(u) = Q K_u^T. A K slot is released when its
// QK^T completes, a V slot when its PV completes.
template <class C>
__device__ void attn_mma_role_split(const AttnParams& p, const TileInfo t0, const TileInfo t1, uint8_t* sQ,
                                    uint8_t* sK, uint8_t* sV, AttnMisc* misc, uint32_t tmem, const Waiter w) {
  using namespace ptx;
  constexpr uint32_t FULL = 0xffffffffu;
  const bool leader = elect_one();
  const uint32_t s_col[2] = {0u, 128u};
  const uint32_t o_col[2] = {256u, 256u + C::DV};
  const uint32_t hi = desc_hi(1024, 2);
  const uint32_t q_lo = desc_lo(smem_addr(sQ), 16);
  const uint32_t k_lo0 = desc_lo(smem_addr(sK), 16);
  const uint32_t v_lo0 = desc_lo(smem_addr(sV), C::CHUNK_BYTES);
  int pend[2] = {-1, -1};  // V slot of the warpgroup's pending PV
  uint32_t pend_ph[2] = {0u, 0u};
  int pv_cnt[2] = {0, 0};
  int k_it = 0, v_it = 0;
  const int n = t0.n_kv;
  bool ok = __all_sync(FULL, w.wait(smem_addr(&misc->q_full), 0));
  tc_fence_after();
  auto issue_pending_pv = [&](int x) {
    if (pend[x] < 0) return;
    if (!(ok = __all_sync(FULL, w.wait(smem_addr(&misc->p_full[x]), pv_cnt[x] & 1)))) return;
    if (!(ok = __all_sync(FULL, w.wait(smem_addr(&misc->kv_full[C::K_STAGES + pend[x]]), pend_ph[x])))) return;
    tc_fence_after();
    if (leader) {
      issue_pv<C>(tmem + o_col[x], tmem + s_col[x], v_lo0 + pend[x] * (C::V_TILE >> 4), hi, pv_cnt[x] > 0);
      tc_commit(smem_addr(&misc->kv_empty[C::K_STAGES + pend[x]]));  // V slot free once the PV finishes
    }
    __syncwarp();
    ++pv_cnt[x];
    pend[x] = -1;
  };
  for (int u = next_kept_tile<C>(p, misc, 3, t0.u0, n); u < n && ok; u = next_kept_tile<C>(p, misc, 3, u + 1, n)) {
    const int x = keep_tile<C>(p, t1, u, misc) ? 1 : 0;
    issue_pending_pv(x);
    if (!ok) break;
    const int ks = k_it % C::K_STAGES;
    const uint32_t kph = (k_it / C::K_STAGES) & 1;
    ++k_it;
    if (!(ok = __all_sync(FULL, w.wait(smem_addr(&misc->kv_full[ks]), kph)))) break;
    tc_fence_after();
    if (leader) {
      issue_qk<C>(tmem + s_col[x], q_lo, k_lo0 + ks * (C::K_TILE >> 4), hi);
      tc_commit(smem_addr(&misc->s_full[x]));
      tc_commit(smem_addr(&misc->kv_empty[ks]));  // K slot free once S_x(u) finishes
    }
    __syncwarp();
    pend[x] = v_it % C::V_STAGES;
    pend_ph[x] = (v_it / C::V_STAGES) & 1;
    ++v_it;
  }
  for (int x = 0; x < 2 && ok; ++x) issue_pending_pv(x);
  if (leader) {
    if (ok) tc_commit(smem_addr(&misc->o_full));
    tc_commit(smem_addr(&misc->drain));
  }
  __syncwarp();
  w.drain(smem_addr(&misc->drain), 0);
}

// Shared-memory P: O += P V with P (A operand, K-major, 128-byte swizzle)
// read from shared memory. K-steps of 32 keys advance 32 bytes in the row.
template <class C>
__device__ __forceinline__ void issue_pv_ss(uint32_t tmem_o, uint32_t p_lo, uint32_t v_lo, uint32_t hi,
                                            uint32_t accumulate) {
#pragma unroll
  for (int s = 0; s < C::PV_STEPS; ++s)
    ptx::mma_ss_f8_lean_acc(tmem_o, p_lo + ((s * 32) >> 4), hi, v_lo + ((s * C::PV_K * 128) >> 4), hi,
                            C::IDESC_PV, s > 0 ? 1u : accumulate);
}

// MMA issue for split tiles with P in shared memory (E4M3 P). Per pair of kept
// tiles (a for warpgroup 0, b for warpgroup 1): QK^T of the NEXT pair as soon as
// each softmax has loaded its current S (s_free), then PV_0(a), PV_1(b) once
// their P is in shared memory (p_full), committed to pv_done[x].
template <class C>
__device__ void attn_mma_role_psmem_split(const AttnParams& p, const TileInfo t0, uint8_t* sQ, uint8_t* sP0,
                                          uint8_t* sP1, uint8_t* sK, uint8_t* sV, AttnMisc* misc, uint32_t tmem,
                                          const Waiter w) {
  using namespace ptx;
  constexpr uint32_t FULL = 0xffffffffu;
  const bool leader = elect_one();
  const uint32_t hi = desc_hi(1024, 2);
  const uint32_t q_lo = desc_lo(smem_addr(sQ), 16);
  const uint32_t p_lo[2] = {desc_lo(smem_addr(sP0), 16), desc_lo(smem_addr(sP1), 16)};
  const uint32_t k_lo0 = desc_lo(smem_addr(sK), 16);
  const uint32_t v_lo0 = desc_lo(smem_addr(sV), C::CHUNK_BYTES);
  const uint32_t s_col[2] = {0u, 128u};
  const uint32_t o_col[2] = {256u, 256u + C::DV};
  const int n = t0.n_kv;
  int s_cnt[2] = {0, 0}, pv_cnt[2] = {0, 0};
  int k_it = 0, v_it = 0;
  bool ok = __all_sync(FULL, w.wait(smem_addr(&misc->q_full), 0));
  tc_fence_after();
  auto next = [&](int from) { return next_kept_tile<C>(p, misc, 3, from, n); };
  // S_x(u) into warpgroup x's S columns, from the next K slot.
  auto issue_s = [&](int x) {
    const int ks = k_it % C::K_STAGES;
    const uint32_t kph = (k_it / C::K_STAGES) & 1;
    ++k_it;
    if (s_cnt[x] > 0) {  // the softmax must have loaded this warpgroup's previous S
      if (!(ok = __all_sync(FULL, w.wait(smem_addr(&misc->s_free[x]), (s_cnt[x] - 1) & 1)))) return;
    }
    if (!(ok = __all_sync(FULL, w.wait(smem_addr(&misc->kv_full[ks]), kph)))) return;
    tc_fence_after();
    if (leader) {
      issue_qk<C>(tmem + s_col[x], q_lo, k_lo0 + ks * (C::K_TILE >> 4), hi);
      tc_commit(smem_addr(&misc->s_full[x]));
      tc_commit(smem_addr(&misc->kv_empty[ks]));
    }
    __syncwarp();
    ++s_cnt[x];
  };
  // O_x += P_x V from the next V slot, once the softmax has written P_x.
  auto issue_pv = [&](int x) {
    const int vs = v_it % C::V_STAGES;
    const uint32_t vph = (v_it / C::V_STAGES) & 1;
    ++v_it;
    if (!(ok = __all_sync(FULL, w.wait(smem_addr(&misc->p_full[x]), pv_cnt[x] & 1)))) return;
    if (!(ok = __all_sync(FULL, w.wait(smem_addr(&misc->kv_full[C::K_STAGES + vs]), vph)))) return;
    tc_fence_after();
    if (leader) {
      issue_pv_ss<C>(tmem + o_col[x], p_lo[x], v_lo0 + vs * (C::V_TILE >> 4), hi, pv_cnt[x] > 0);
      tc_commit(smem_addr(&misc->pv_done[x]));
      tc_commit(smem_addr(&misc->kv_empty[C::K_STAGES + vs]));
    }
    __syncwarp();
    ++pv_cnt[x];
  };
  int ua = next(t0.u0);
  int ub = ua < n ? next(ua + 1) : n;
  if (ua < n && ok) issue_s(0);
  if (ub < n && ok) issue_s(1);
  while (ua < n && ok) {
    const int na = ub < n ? next(ub + 1) : n;
    const int nb = na < n ? next(na + 1) : n;
    if (na < n) issue_s(0);
    if (nb < n && ok) issue_s(1);
    if (!ok) break;
    issue_pv(0);
    if (ub < n && ok) issue_pv(1);
    ua = na;
    ub = nb;
  }
  if (leader) tc_commit(smem_addr(&misc->drain));
  __syncwarp();
  w.drain(smem_addr(&misc->drain), 0);
}

// MMA issue for the shared-memory-P pipeline. Per kept KV tile u (in order):
//   QK^T of the NEXT kept tile for each query tile, as soon as that tile's
//   softmax has loaded its current S (s_free) -- this overlaps the softmax;
//   then PV of tile u once P_x(u) is in shared memory (p_full), committed to
//   pv_done[x], which the softmax waits on before it rewrites P or O.
template <class C>
__device__ void attn_mma_role_psmem(const AttnParams& p, const TileInfo t0, const TileInfo t1, int b, int hkv,
                                    uint8_t* sQ0, uint8_t* sQ1, uint8_t* sP0, uint8_t* sP1, uint8_t* sSlots,
                                    AttnMisc* misc, uint32_t tmem, const Waiter w) {
  using namespace ptx;
  constexpr uint32_t FULL = 0xffffffffu;
  const bool leader = elect_one();
  const uint32_t hi = desc_hi(1024, 2);
  const uint32_t q_lo0 = desc_lo(smem_addr(sQ0), 16), q_lo1 = desc_lo(smem_addr(sQ1), 16);
  const uint32_t p_lo0 = desc_lo(smem_addr(sP0), 16), p_lo1 = desc_lo(smem_addr(sP1), 16);
  const uint32_t k_lo0 = desc_lo(smem_addr(sSlots), 16);
  const uint32_t v_lo0 = desc_lo(smem_addr(sSlots), C::CHUNK_BYTES);
  const uint32_t s_col[2] = {0u, 128u};
  const uint32_t o_col[2] = {256u, 256u + C::DV};
  const int n_u = max(t0.n_kv, t1.n_kv);
  int s_cnt[2] = {0, 0}, pv_cnt[2] = {0, 0};
  int slot_it = 0;
  bool ok = __all_sync(FULL, w.wait(smem_addr(&misc->q_full), 0));
  tc_fence_after();
  auto next_kept = [&](int from) { return next_kept_tile<C>(p, misc, 3, from, n_u); };
  // S_x(u) = Q_x K_u^T into tile x's S columns; K_u lives in slot ks.
  auto issue_s = [&](int x, int u, int ks) {
    if (!keep_tile<C>(p, x ? t1 : t0, u, misc)) return;
    if (s_cnt[x] > 0) {  // the softmax must have loaded this tile's previous S
      if (!(ok = __all_sync(FULL, w.wait(smem_addr(&misc->s_free[x]), (s_cnt[x] - 1) & 1)))) return;
      tc_fence_after();
    }
    if (leader) {
      issue_qk<C>(tmem + s_col[x], x ? q_lo1 : q_lo0, k_lo0 + ks * (C::SLOT >> 4), hi);
      tc_commit(smem_addr(&misc->s_full[x]));
    }
    __syncwarp();
    ++s_cnt[x];
  };
  // O_x += P_x V (V in slot vsl), once the softmax has written P_x; committed
  // to pv_done[x].
  auto issue_pv = [&](int x, int vsl) {
    if (!(ok = __all_sync(FULL, w.wait(smem_addr(&misc->p_full[x]), pv_cnt[x] & 1)))) return;
    tc_fence_after();
    if (leader) {
      const uint32_t plo = x ? p_lo1 : p_lo0;
      const uint32_t vlo = v_lo0 + vsl * (C::SLOT >> 4);
      issue_pv_ss<C>(tmem + o_col[x], plo, vlo, hi, pv_cnt[x] > 0);
      if constexpr (C::P2) issue_pv_ss<C>(tmem + o_col[x], plo + (C::P_TILE >> 4), vlo, hi, 1u);
      tc_commit(smem_addr(&misc->pv_done[x]));
    }
    __syncwarp();
    ++pv_cnt[x];
  };
  auto release = [&](int slot) {
    if (leader) tc_commit(smem_addr(&misc->kv_empty[slot]));  // arrives when the MMAs issued so far finish
    __syncwarp();
  };
  int u = next_kept(min(t0.u0, t1.u0));
  int vs = 0;
  if (u < n_u && ok) {
    const int ks = slot_it % C::STAGES;
    const uint32_t kph = (slot_it / C::STAGES) & 1;
    ++slot_it;
    vs = slot_it % C::STAGES;
    ++slot_it;
    if ((ok = __all_sync(FULL, w.wait(smem_addr(&misc->kv_full[ks]), kph)))) {
      tc_fence_after();
      issue_s(0, u, ks);
      if (ok) issue_s(1, u, ks);
      if (ok) release(ks);
    }
  }
  // Per kept KV tile u: QK^T of the next kept tile for both query tiles (as
  // soon as each softmax has loaded its current S), then PV of tile u for
  // both. (Issuing in the order the two softmax warpgroups release -- tile 1's
  // PV one tile behind -- was measured 7 % slower with a BF16 QK^T.)
  while (u < n_u && ok) {
    const uint32_t vph = ((slot_it - 1) / C::STAGES) & 1;  // ring phase of V_u (slot vs)
    const int nu = next_kept(u + 1);
    int nks = 0, nvs = 0;
    if (nu < n_u) {
      nks = slot_it % C::STAGES;
      const uint32_t nkph = (slot_it / C::STAGES) & 1;
      ++slot_it;
      nvs = slot_it % C::STAGES;
      ++slot_it;
      if (!(ok = __all_sync(FULL, w.wait(smem_addr(&misc->kv_full[nks]), nkph)))) break;
      tc_fence_after();
      issue_s(0, nu, nks);
      if (ok) issue_s(1, nu, nks);
      if (!ok) break;
      release(nks);  // K_nu: both S MMAs issued
    }
    if (!(ok = __all_sync(FULL, w.wait(smem_addr(&misc->kv_full[vs]), vph)))) break;
    tc_fence_after();
    if (keep_tile<C>(p, t0, u, misc)) {
      issue_pv(0, vs);
      if (!ok) break;
    }
    if (keep_tile<C>(p, t1, u, misc)) {
      issue_pv(1, vs);
      if (!ok) break;
    }
    release(vs);  // V_u: both PV MMAs issued
    u = nu;
    vs = nvs;
  }
  if (leader) tc_commit(smem_addr(&misc->drain));
  __syncwarp();
  w.drain(smem_addr(&misc->drain), 0);
}

// 2^x on the FMA pipe, for two values at once ("FlashInfer FP8/BF16
// mixed-precision attention for Blackwell", section 3: part of the exp2 work
// moved from MUFU to FMA). x is clamped to [-125, +inf) (results below 2^-125
// are zero to every P format); n = rint(x) comes from adding 1.5 * 2^23 (the
// integer lands in the low mantissa bits), f = x - n lies in [-1/2, 1/2],
// 2^f is a polynomial in f fitted to minimise the relative error on that
// interval (degree 2: 1.7e-3, degree 3: 7.5e-5), and 2^n is added to the
// exponent field as an integer (n << 23). Valid for x < 128.
// Share of a tile's exponentials taken by the polynomial: one group of four
// scores in kExpPolyEvery (0: none). A standalone exp + pack pass ran 16 %
// faster with one in four, but in the kernel every such setting measured
// slower (3-6 % for the E4M3-P modes): the softmax chain, not MUFU, bounds the
// kernel, and with one E4M3 term the polynomial's rounding differs from MUFU's
// for the weight the row-sum correction below relies on. Kept selectable.
constexpr int kExpPolyEvery = 0;

template <int DEG>
__device__ __forceinline__ void exp2_poly_x2(float& a, float& b) {
  using namespace ptx;
  a = fmaxf(a, -125.f);
  b = fmaxf(b, -125.f);
  float ja, jb, na, nb, fa, fb, pa, pb;
  fadd2(ja, jb, a, b, 12582912.f, 12582912.f);
  fadd2(na, nb, ja, jb, -12582912.f, -12582912.f);
  fadd2(fa, fb, a, b, -na, -nb);
  if constexpr (DEG == 3) {
    ffma2(pa, pb, fa, fb, 0.05517098f, 0.05517098f, 0.24260971f, 0.24260971f);
    ffma2(pa, pb, pa, pb, fa, fb, 0.69326097f, 0.69326097f);
    ffma2(pa, pb, pa, pb, fa, fb, 0.99992818f, 0.99992818f);
  } else {
    ffma2(pa, pb, fa, fb, 0.23842251f, 0.23842251f, 0.70343643f, 0.70343643f);
    ffma2(pa, pb, pa, pb, fa, fb, 1.00044274f, 1.00044274f);
  }
  a = __int_as_float(__float_as_int(pa) + (__float_as_int(ja) << 23));
  b = __int_as_float(__float_as_int(pb) + (__float_as_int(jb) << 23));
}

// ------------------------------------------------------- narrow softmax ----
// Decode tiles whose packed rows are all in rows 0..15 (Sq * group <= 16, BF16
// P in TMEM): only the first warp of the warpgroup (TMEM lanes 0..31) holds
// valid rows. It loads S with the 16-lane shape, which spreads rows 0..7 and
// 8..15 over all 32 threads (thread t: rows t/4 and 8 + t/4, key pairs
// 8k + 2(t%4), k = 0..15), so each thread exponentiates 32 (or 64) scores
// instead of a row of 128 of which only 8 or 16 rows are real. The row max
// and sum are reduced over the four threads of a row; P goes back over S with
// the 16-lane x 128-bit shape, whose column 4k + t%4 is exactly the pair of
// keys thread t holds. The other three warps only keep the barrier count.
// Returns, for the epilogue, m and l of row `lane` (lanes 0..15), and the
// number of tiles processed.
template <class C>
__device__ void attn_softmax_narrow(const AttnParams& p, const TileInfo t, int x, AttnMisc* misc, uint32_t tmem,
                                    float cq, const Waiter w, float& m_out, float& l_out, int& it_out, bool& ok_out) {
  using namespace ptx;
  constexpr uint32_t FULL = 0xffffffffu;
  const int warp = (threadIdx.x >> 5) & 3;
  const int lane = threadIdx.x & 31;
  const int j = lane & 3, rr = lane >> 2;
  const uint32_t tS = tmem + (x ? 128u : 0u);                 // lane quadrant 0
  const uint32_t tO = tmem + (x ? 256u + C::DV : 256u);
  const int nh = p.n_rows > 8 ? 2 : 1;                         // row halves with valid rows
  constexpr float tau = 8.f;                                   // BF16 P
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  int it = 0;
  bool ok = true;
  for (int u = next_kept_tile<C>(p, misc, 1 << t.x, t.u0, t.n_kv); u < t.n_kv;
       u = next_kept_tile<C>(p, misc, 1 << t.x, u + 1, t.n_kv)) {
    ok = __all_sync(FULL, w.wait(smem_addr(&misc->s_full[x]), it & 1)) && ok;
    if (!ok) break;
    tc_fence_after();
    if (warp == 0) {
      uint32_t sr[64];
      tmem_ld_16x256b_x16(tS, sr);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 64; q += 32) {
        uint32_t (&blk)[32] = *reinterpret_cast<uint32_t (*)[32]>(&sr[q]);
        reg_fence(blk);
      }
      float alpha[2] = {1.f, 1.f};
      bool resc = false;
      uint32_t pk[32];  // P columns 4k + j of row rr (2k) and 8 + rr (2k + 1)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // keys at or past lim are hidden for this row (ragged end, causal)
        const int row = rr + 8 * h;
        const int tok = t.tok0 + (row >> p.group_shift);
        int lim = p.Skv - u * C::BN;
        if (p.causal) lim = min(lim, tok + 1 + (p.Skv - p.Sq) - u * C::BN);
        if (h >= nh || tok >= p.Sq) lim = 0;  // a padding row: all hidden
        float f[32];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          f[2 * k] = 8 * k + 2 * j < lim ? __uint_as_float(sr[4 * k + 2 * h]) : -INFINITY;
          f[2 * k + 1] = 8 * k + 2 * j + 1 < lim ? __uint_as_float(sr[4 * k + 2 * h + 1]) : -INFINITY;
        }
        float mt = f[0];
#pragma unroll
        for (int i = 1; i < 32; ++i) mt = fmaxf(mt, f[i]);
        mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 1));
        mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 2));
        mt *= cq;
        const float m_new = fmaxf(m[h], mt);
        if (it == 0) {
          m[h] = m_new;
        } else if (m_new > m[h] + tau) {
          alpha[h] = ex2(m[h] - m_new);
          resc = true;
          m[h] = m_new;
        }
        const float nmb = -(m[h] == -INFINITY ? 0.f : m[h]);
        float rs = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          float e0, e1;
          ffma2(e0, e1, f[2 * k], f[2 * k + 1], cq, cq, nmb, nmb);
          e0 = ex2(e0);
          e1 = ex2(e1);
          pk[2 * k + h] = pack_bf16x2(e0, e1);
          rs += e0 + e1;
        }
        l[h] = l[h] * alpha[h] + rs;
      }
      // Lazy O correction (rows rr and 8 + rr of this thread), before P is
      // released: the arrival of S proved the previous PV finished.
      if (__any_sync(FULL, resc)) {
        uint32_t o[64];
        tmem_ld_16x256b_x16(tO, o);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 64; q += 32) {
          uint32_t (&blk)[32] = *reinterpret_cast<uint32_t (*)[32]>(&o[q]);
          reg_fence(blk);
        }
#pragma unroll
        for (int k = 0; k < 16; ++k)
#pragma unroll
          for (int e = 0; e < 4; ++e) o[4 * k + e] = __float_as_uint(__uint_as_float(o[4 * k + e]) * alpha[e >> 1]);
        tmem_st_16x256b_x16(tO, o);
      }
      tmem_st_16x128b_x16(tS, pk);
      tmem_wait_st();
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&misc->p_full[x]));
    ++it;
  }
  // Row totals (four threads per row), then row `lane` for the epilogue.
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l[h] += __shfl_xor_sync(FULL, l[h], 1);
    l[h] += __shfl_xor_sync(FULL, l[h], 2);
  }
  const int src = 4 * (lane & 7);
  const float m0 = __shfl_sync(FULL, m[0], src), m1 = __shfl_sync(FULL, m[1], src);
  const float l0 = __shfl_sync(FULL, l[0], src), l1 = __shfl_sync(FULL, l[1], src);
  const bool mine = warp == 0 && lane < 8 * nh;
  m_out = mine ? (lane < 8 ? m0 : m1) : -INFINITY;
  l_out = mine ? (lane < 8 ? l0 : l1) : 0.f;
  it_out = it;
  ok_out = ok;
}

// --------------------------------------------------------------- softmax ----
// One thread per query row (TMEM lane = row). Per kept KV tile: load S (128
// fp32 or s32 per row) from TMEM, scale and mask, exponentiate with packed
// fp32x2 FMAs feeding MUFU ex2, pack P (BF16 into TMEM over S, or E4M3 into
// shared memory) and release it to the MMA warp with one arrive per warp.
//
// The running row max m is lazy ("FlashInfer FP8/BF16 mixed-precision
// attention for Blackwell", section 3): it only moves, and O and l are only
// rescaled, when a tile's max exceeds m by more than tau (log2 units). Each
// tile takes its row max first, then one pass computes the exponentials,
// packs P and adds the row sum. (Loading the next tile's S from TMEM while
// this tile's E4M3 P is stored was measured 10 % slower.)
template <class C>
__device__ void attn_softmax_role(const AttnParams& p, const TileInfo t, int x, int b, int hkv, uint8_t* sQx,
                                  uint8_t* sPx, uint8_t* sX, int n_turns, AttnMisc* misc, uint32_t tmem,
                                  const CUtensorMap* tmO, const Waiter w) {
  using namespace ptx;
  constexpr uint32_t FULL = 0xffffffffu;
  constexpr int NCH = C::BN / 32;  // 32-key chunks per tile (one TMEM load each)
  constexpr int OB = C::DV / 32;   // 32-column blocks of O
  const int warp = (threadIdx.x >> 5) & 3;  // TMEM lane quadrant of this warp
  const int lane = threadIdx.x & 31;
  const int r = warp * 32 + lane;  // row within the tile
  // Query token and head of this row (packed: row r = token r >> shift, head r & (group - 1)).
  const int row = C::PACKED ? t.tok0 + (r >> p.group_shift) : t.q0 + r;
  const int head = C::PACKED ? t.h + (r & ((1 << p.group_shift) - 1)) : t.h;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tS = tmem + lane_off + (x ? 128u : 0u);
  const uint32_t tO = tmem + lane_off + (x ? 256u + C::DV : 256u);
  const bool lead = (threadIdx.x & 127) == 0;  // one thread of the query tile
  const int64_t bhq = static_cast<int64_t>(b) * p.Hq + head;
  const int64_t bhk = static_cast<int64_t>(b) * p.Hkv + hkv;

  // Row factor: softmax scale * log2(e) * Q scale of this row.
  float cq = p.scale_log2;
  if (C::QK != QK_BF16) cq *= sf_lookup(p.sf_q, p.sf_q_kind, bhq, p.sf_q_nblk, min(row, p.Sq - 1), p.sf_q_rpb);
  const float ck_uniform =
      p.sf_k_kind == FMHA_SF_PER_TOKEN_BLOCK ? 1.f : sf_lookup(p.sf_k, p.sf_k_kind, bhk, 1, 0, 1);
  const bool ck_blocked = C::QK != QK_BF16 && p.sf_k_kind == FMHA_SF_PER_TOKEN_BLOCK;

  // P encoding: E4M3 P holds p * g with g = 1 / sf_p; the lazy-rescale
  // threshold tau keeps the stale-max bound 2^tau * g <= 448. BF16 P: g = 1, tau = 8.
  float log2g = 0.f;
  float tau = 8.f;
  if constexpr (C::PV == PV_E4M3) {
    float sfp = 1.f / 16.f;
    if (p.sf_p_kind == FMHA_SF_PER_TENSOR) sfp = p.sf_p[0];
    if (p.sf_p_kind == FMHA_SF_PER_TOKEN_BLOCK) sfp = p.sf_p[bhq * p.sf_p_nblk + t.tok0 / p.sf_p_rpb];
    log2g = -__log2f(sfp);
    tau = fminf(8.f, fmaxf(0.f, floorf(__log2f(448.f * sfp))));
  }

  // K scale of each 32-key chunk of tile u (token-block K scales).
  auto load_ck = [&](int u, float (&dst)[NCH]) {
#pragma unroll
    for (int c = 0; c < NCH; ++c)
      dst[c] = (ck_blocked ? __ldg(p.sf_k + bhk * p.sf_k_nblk + min(u * C::BN + 32 * c, p.Skv - 1) / p.sf_k_rpb)
                           : ck_uniform) * cq;
  };

  float m = -INFINITY;  // running row max (log2 units, scaled)
  float l = 0.f;        // running row sum of P (times g)
  int it = 0;
  bool ok = true;
  bool narrow = false;  // decode tiles of at most 16 rows: the narrow pass above
  if constexpr (C::PACKED && C::PV == PV_BF16) {
    if (p.narrow) {
      attn_softmax_narrow<C>(p, t, x, misc, tmem, cq * ck_uniform, w, m, l, it, ok);
      narrow = true;
    }
  }
  for (int u = narrow ? t.n_kv : next_kept_tile<C>(p, misc, 1 << t.x, t.u0, t.n_kv); u < t.n_kv;
       u = next_kept_tile<C>(p, misc, 1 << t.x, u + 1, t.n_kv)) {
    float ck[NCH];
    load_ck(u, ck);  // issued before the wait: the loads overlap it
    ok = __all_sync(FULL, w.wait(smem_addr(&misc->s_full[x]), it & 1)) && ok;
    if (!ok) break;
    tc_fence_after();
    int lim = p.Skv - u * C::BN;  // keys at or past `lim` in this tile are hidden
    if (p.causal) lim = min(lim, row + 1 + (p.Skv - p.Sq) - u * C::BN);

    // S of this tile into f (fp32 scores; hidden keys -inf).
    float f[NCH][32];
    {
      uint32_t s[NCH][32];
#pragma unroll
      for (int c = 0; c < NCH; ++c) tmem_ld32(tS + 32 * c, s[c]);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < NCH; ++c) reg_fence(s[c]);
      if constexpr (C::PSMEM) {  // S is in registers: the MMA warp may issue the next QK^T into this tile
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&misc->s_free[x]));
      }
      // INT8 scores: s32 s is exact in fp32 (|s| <= 127 * 127 * D < 2^22): one
      // integer add makes the bits of 1.5 * 2^23 + s, one exact subtraction
      // (two per packed instruction) removes the offset.
#pragma unroll
      for (int c = 0; c < NCH; ++c)
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          if constexpr (C::QK == QK_INT8)
            fadd2(f[c][j], f[c][j + 1], __int_as_float(static_cast<int>(s[c][j]) + 0x4B400000),
                  __int_as_float(static_cast<int>(s[c][j + 1]) + 0x4B400000), -12582912.f, -12582912.f);
          else
            f[c][j] = __uint_as_float(s[c][j]), f[c][j + 1] = __uint_as_float(s[c][j + 1]);
        }
    }
    if (lim < C::BN) {
#pragma unroll
      for (int c = 0; c < NCH; ++c)
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (32 * c + j >= lim) f[c][j] = -INFINITY;
    }

    // Row max of the tile (ck > 0: the scaled max is the raw max times ck).
    float m_tile = -INFINITY;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      float a0 = fmax3(f[c][0], f[c][1], f[c][2]), a1 = fmax3(f[c][3], f[c][4], f[c][5]);
#pragma unroll
      for (int j = 6; j < 30; j += 4) {
        a0 = fmax3(a0, f[c][j], f[c][j + 1]);
        a1 = fmax3(a1, f[c][j + 2], f[c][j + 3]);
      }
      m_tile = fmaxf(m_tile, fmax3(a0, a1, fmaxf(f[c][30], f[c][31])) * ck[c]);
    }
    const float m_new = fmaxf(m, m_tile);
    float alpha = 1.f;
    bool resc = false;
    if (it == 0) {
      m = m_new;
    } else if (m_new > m + tau) {
      alpha = ex2(m - m_new);
      resc = true;
      m = m_new;
    }
    // Lazy O correction (whole warp: tcgen05.ld/st are warp-wide). With P in
    // TMEM the arrival of S proved the previous PV finished; with P in shared
    // memory the previous PV may still run, so it is done after pv_done below.
    auto rescale_o = [&]() {
      if (__any_sync(FULL, resc)) {
#pragma unroll 1
        for (int c = 0; c < OB; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * c, o);
          tmem_wait_ld();
          reg_fence(o);
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
          tmem_st32(tO + 32 * c, o);
        }
      }
    };
    if constexpr (!C::PSMEM) rescale_o();
    // Row r of the 128 x 128-byte E4M3 P tile in shared memory, 16-byte chunks
    // XOR-swizzled by r % 8 (the 128-byte swizzle the PV descriptor expects).
    // (Storing each chunk inside the exp pass was measured 15 % slower: the
    // stores then compete with the turn's exponentials.)
    [[maybe_unused]] const uint32_t prow = smem_addr(sPx) + r * 128;
    [[maybe_unused]] auto store_p = [&](int k, uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, uint32_t plane) {
      const uint32_t addr = prow + plane + ((k ^ (r & 7)) << 4);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w0), "r"(w1), "r"(w2), "r"(w3)
                   : "memory");
    };

    // Turn-taking on the exp2 unit: for the first n_turns tiles (both tiles
    // walk the same KV tiles) the warpgroups alternate their exponential
    // phases, so that one exponentiates while the other loads, reduces and
    // stores. Tile 0 goes first.
    if (C::TURNS && (x == 0 ? (it >= 1 && it < n_turns) : (it < n_turns))) {
      ok = __all_sync(FULL, w.wait(smem_addr(&misc->exp_done[x ^ 1]), (x == 0 ? it - 1 : it) & 1)) && ok;
#pragma unroll
      for (int c = 0; c < NCH; ++c) reg_fence(f[c]);
    }

    // Exponentials, P and its row sum in one pass: per group of scores
    // 2^(f * ck - mb) (packed FMAs feeding MUFU ex2), packed to BF16 (TMEM)
    // or E4M3 (registers, for shared memory) as soon as a group is done, so
    // the conversions and additions fill the issue slots between ex2s.
    const float nmb = -((m == -INFINITY ? 0.f : m) - log2g);
    float rs = 0.f;
    [[maybe_unused]] uint32_t pk[C::PV == PV_E4M3 ? 8 * NCH : 1];
    [[maybe_unused]] uint32_t pl[C::P2 ? 8 * NCH : 1];
    if constexpr (C::PV == PV_BF16) {
      // BF16 P of keys 64q..64q+63 goes over TMEM columns [32q, 32q + 32) of S.
      float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f;
#pragma unroll
      for (int q = 0; q < NCH / 2; ++q) {
        uint32_t p32[32];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int c = 2 * q + h;
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            float e0, e1, e2, e3;
            ffma2(e0, e1, f[c][j], f[c][j + 1], ck[c], ck[c], nmb, nmb);
            ffma2(e2, e3, f[c][j + 2], f[c][j + 3], ck[c], ck[c], nmb, nmb);
            e0 = ex2(e0); e1 = ex2(e1); e2 = ex2(e2); e3 = ex2(e3);
            p32[16 * h + j / 2] = pack_bf16x2(e0, e1);
            p32[16 * h + j / 2 + 1] = pack_bf16x2(e2, e3);
            fadd2(r0, r1, r0, r1, e0, e1);
            fadd2(r2, r3, r2, r3, e2, e3);
          }
        }
        tmem_st32(tS + 32 * q, p32);
      }
      rs = (r0 + r1) + (r2 + r3);
    } else if constexpr (C::P2) {
      // Two-term E4M3 P: hi = E4M3(p g), lo = E4M3(p g - hi) (the residual taken
      // in f16), ~7 significant bits between them; both feed their own PV
      // product. The row sum adds the unrounded values (as precise as BF16 P).
      // With kExpPolyEvery set, the degree-3 polynomial (well inside the two
      // terms' precision) takes that share of the exponentials.
      float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f;
#pragma unroll
      for (int c = 0; c < NCH; ++c)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float e[4];
          ffma2(e[0], e[1], f[c][4 * j], f[c][4 * j + 1], ck[c], ck[c], nmb, nmb);
          ffma2(e[2], e[3], f[c][4 * j + 2], f[c][4 * j + 3], ck[c], ck[c], nmb, nmb);
          if (kExpPolyEvery > 0 && j % kExpPolyEvery == kExpPolyEvery - 1) {
            exp2_poly_x2<3>(e[0], e[1]);
            exp2_poly_x2<3>(e[2], e[3]);
          } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) e[q] = ex2(e[q]);
          }
          const uint32_t h01 = pack_e4m3x2(e[0], e[1]), h23 = pack_e4m3x2(e[2], e[3]);
          pk[c * 8 + j] = h01 | (h23 << 16);
          const uint32_t d01 = hsub2(pack_f16x2(e[0], e[1]), e4m3x2_to_f16x2(h01));
          const uint32_t d23 = hsub2(pack_f16x2(e[2], e[3]), e4m3x2_to_f16x2(h23));
          pl[c * 8 + j] = f16x2_to_e4m3x2(d01) | (f16x2_to_e4m3x2(d23) << 16);
          fadd2(r0, r1, r0, r1, e[0], e[1]);
          fadd2(r2, r3, r2, r3, e[2], e[3]);
        }
      rs = (r0 + r1) + (r2 + r3);
    } else {
      // One E4M3 term. The row sum adds the unrounded values (packed adds; the
      // conversions back from E4M3 cost 3-5 % of the kernel) plus, below, the
      // rounding error of the tile's largest weight: a dominant key's
      // normalised weight is then exact, as with a sum of the stored values
      // (an outlier value otherwise comes back off by up to 2^-4 of itself).
      // The correction recomputes that weight with the same MUFU ex2, so it is
      // bit-identical to the stored one; a polynomial exponential would break
      // that, so this mode always uses MUFU.
      float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f;
#pragma unroll
      for (int c = 0; c < NCH; ++c)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float e0, e1, e2, e3;
          ffma2(e0, e1, f[c][4 * j], f[c][4 * j + 1], ck[c], ck[c], nmb, nmb);
          ffma2(e2, e3, f[c][4 * j + 2], f[c][4 * j + 3], ck[c], ck[c], nmb, nmb);
          e0 = ex2(e0); e1 = ex2(e1); e2 = ex2(e2); e3 = ex2(e3);
          pk[c * 8 + j] = pack_e4m3x2(e0, e1) | (pack_e4m3x2(e2, e3) << 16);
          fadd2(r0, r1, r0, r1, e0, e1);
          fadd2(r2, r3, r2, r3, e2, e3);
        }
      rs = (r0 + r1) + (r2 + r3);
      if (m_tile != -INFINITY) {
        const float emax = ex2(m_tile + nmb);
        rs += e4m3_round(emax) - emax;
      }
    }
    if (C::TURNS && (x == 0 ? (it < n_turns) : (it + 1 < n_turns))) {
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&misc->exp_done[x]));
    }
    if constexpr (C::PSMEM) {
      // The previous PV must be done before P (single buffer) or O is rewritten.
      if (it > 0) {
        ok = __all_sync(FULL, w.wait(smem_addr(&misc->pv_done[x]), (it - 1) & 1)) && ok;
        tc_fence_after();
      }
      rescale_o();
#pragma unroll
      for (int k = 0; k < 2 * NCH; ++k) {
        store_p(k, pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3], 0);
        if constexpr (C::P2) store_p(k, pl[4 * k], pl[4 * k + 1], pl[4 * k + 2], pl[4 * k + 3], C::P_TILE);
      }
      fence_proxy_async_smem();  // generic-proxy P writes -> tensor-core reads
    }
    l = l * alpha + rs;
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();  // the warp's P stores are ordered before lane 0's arrive
    if (lane == 0) mbar_arrive(smem_addr(&misc->p_full[x]));
    ++it;
  }

  // ---- epilogue ----
  bool have_o = false;
  if (ok) ok = __all_sync(FULL, w.wait(smem_addr(&misc->q_full), 0));  // Q buffer (our staging) has landed
  if (ok && it > 0) {  // the last PV product has finished
    if constexpr (C::PSMEM)
      ok = __all_sync(FULL, w.wait(smem_addr(&misc->pv_done[x]), (it - 1) & 1));
    else
      ok = __all_sync(FULL, w.wait(smem_addr(&misc->o_full), 0));
    tc_fence_after();
    have_o = ok;
  }
  float sfv = 1.f;
  if (C::PV == PV_E4M3 && p.sf_v_kind != FMHA_SF_PER_CHANNEL) sfv = sf_lookup(p.sf_v, p.sf_v_kind, bhk, 1, 0, 1);
  const float inv_l = l > 0.f ? sfv / l : 0.f;
  const uint32_t stage0 = smem_addr(sQx);
  constexpr uint32_t TILE_THREADS = 128;
  if constexpr (C::SPLIT) {
    // Split tiles: both warpgroups hold partial results (m, l, O) of the same
    // rows over disjoint keys. Once both have seen their last PV finish, every
    // MMA of the CTA is done and the K/V ring is free: (m, l) per row go
    // through it, and warpgroup x merges and stores columns [64x, 64x + 64):
    // O = (O_0 2^(m_0 - M) + O_1 2^(m_1 - M)) / (l_0 2^(m_0 - M) + l_1 2^(m_1 - M)).
    named_bar_sync(3, 2 * TILE_THREADS);
    float2* ex = reinterpret_cast<float2*>(sX);
    ex[x * 128 + r] = make_float2(have_o ? m : -INFINITY, have_o ? l : -1.f);  // l < 0: no O
    named_bar_sync(3, 2 * TILE_THREADS);
    const float2 e0 = ex[r], e1 = ex[128 + r];
    const bool h0 = e0.y > 0.f, h1 = e1.y > 0.f;
    const float M = fmaxf(h0 ? e0.x : -INFINITY, h1 ? e1.x : -INFINITY);
    const float c0 = h0 ? ex2(e0.x - M) : 0.f, c1 = h1 ? ex2(e1.x - M) : 0.f;
    const float L = (h0 ? e0.y * c0 : 0.f) + (h1 ? e1.y * c1 : 0.f);
    const float inv = L > 0.f ? sfv / L : 0.f;
    // Columns [64x, 64x + 64) of both accumulators (a warpgroup without tiles
    // left its O undefined: its values are selected away, never multiplied).
    const uint32_t tO0 = tmem + lane_off + 256u + 64u * x, tO1 = tO0 + C::DV;
    const uint32_t buf = stage0 + x * C::CHUNK_BYTES;
    const uint32_t base = buf + r * 128;
#pragma unroll 1
    for (int sc = 0; sc < 2; ++sc) {  // 32 columns at a time
      uint32_t o0[32], o1[32];
      tmem_ld32(tO0 + 32 * sc, o0);
      tmem_ld32(tO1 + 32 * sc, o1);
      tmem_wait_ld();
      reg_fence(o0);
      reg_fence(o1);
      auto out_val = [&](int j) {
        const float a = h0 ? __uint_as_float(o0[j]) * c0 : 0.f;
        const float b2 = h1 ? __uint_as_float(o1[j]) * c1 : 0.f;
        float v = (a + b2) * inv;
        if (C::PV == PV_E4M3 && p.sf_v_kind == FMHA_SF_PER_CHANNEL) v *= misc->sf_v[64 * x + 32 * sc + j];
        return v;
      };
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(out_val(2 * j), out_val(2 * j + 1));
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int k = 4 * sc + kk;
        const uint32_t addr = base + ((k ^ (r & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[4 * kk]), "r"(pk[4 * kk + 1]),
                     "r"(pk[4 * kk + 2]), "r"(pk[4 * kk + 3])
                     : "memory");
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(1 + x, TILE_THREADS);
    if (lead && ok) {
      tma_store_4d(tmO, buf, 64 * x, t.h, t.q0, b);
      bulk_commit();
    }
    if (x == 0 && p.lse != nullptr && row < p.Sq && ok)
      p.lse[bhq * p.Sq + row] = L > 0.f ? (M + __log2f(L) - log2g) * 0.69314718055994531f : -INFINITY;
    if (lead) bulk_wait0();
    return;
  }
  if constexpr (C::O8) {
    // E4M3 output: the whole 128-column row is 128 bytes, one swizzled
    // 128 x 128-byte chunk (the size and layout of a 64-column BF16 chunk),
    // written by one TMA store. Column c of the row is O[c] / l * sf_v / sf_o.
    const float inv_lo = inv_l / (p.sf_o != nullptr ? __ldg(p.sf_o) : 1.f);
    const uint32_t base = stage0 + r * 128;
#pragma unroll 1
    for (int sc = 0; sc < C::DV / 32; ++sc) {
      uint32_t o[32];
      if (have_o) {
        tmem_ld32(tO + 32 * sc, o);
        tmem_wait_ld();
        reg_fence(o);
      }
      uint32_t pk[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = 4 * j + e;
          v[e] = have_o ? __uint_as_float(o[col]) * inv_lo : 0.f;
          if (C::PV == PV_E4M3 && p.sf_v_kind == FMHA_SF_PER_CHANNEL) v[e] *= misc->sf_v[32 * sc + col];
        }
        pk[j] = pack_e4m3x2(v[0], v[1]) | (pack_e4m3x2(v[2], v[3]) << 16);
      }
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const uint32_t addr = base + (((2 * sc + kk) ^ (r & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[4 * kk]), "r"(pk[4 * kk + 1]),
                     "r"(pk[4 * kk + 2]), "r"(pk[4 * kk + 3])
                     : "memory");
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(1 + x, TILE_THREADS);
    if (lead && ok) {
      tma_store_4d(tmO, stage0, 0, t.h, t.q0, b);
      bulk_commit();
    }
  }
#pragma unroll 1
  for (int c64 = 0; c64 < (C::O8 ? 0 : C::DV / 64); ++c64) {
    uint32_t o[2][32];
    if (have_o) {
      tmem_ld32(tO + 64 * c64, o[0]);
      tmem_ld32(tO + 64 * c64 + 32, o[1]);
      tmem_wait_ld();
      reg_fence(o[0]);
      reg_fence(o[1]);
    }
    auto out_val = [&](int col) {  // column col (0..63) of this chunk, scaled
      float v = have_o ? __uint_as_float(o[col >> 5][col & 31]) * inv_l : 0.f;
      if (C::PV == PV_E4M3 && p.sf_v_kind == FMHA_SF_PER_CHANNEL) v *= misc->sf_v[64 * c64 + col];
      return v;
    };
    if constexpr (C::PACKED) {
      if (p.n_parts > 1) {  // one partial: O / l in fp32 for the merge kernel (no staging)
        if (row < p.Sq && ok) {
          float* dst = p.o_part + ((((int64_t)t.part * p.B + b) * p.Sq + row) * p.Hq + head) * C::DV + 64 * c64;
#pragma unroll
          for (int j = 0; j < 64; j += 4) {
            asm volatile("st.global.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst + j), "f"(out_val(j)),
                         "f"(out_val(j + 1)), "f"(out_val(j + 2)), "f"(out_val(j + 3))
                         : "memory");
          }
        }
        continue;
      }
    }
    const int buf = c64 % C::O_STAGE_BUFS;
    if (c64 >= C::O_STAGE_BUFS) {  // buffer reuse: the previous store must have read it
      if (lead) bulk_wait_read0();
      named_bar_sync(1 + x, TILE_THREADS);
    }
    const uint32_t base = stage0 + buf * C::CHUNK_BYTES + r * 128;
#pragma unroll
    for (int sc = 0; sc < 2; ++sc) {
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(out_val(32 * sc + 2 * j), out_val(32 * sc + 2 * j + 1));
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int k = 4 * sc + kk;
        const uint32_t addr = base + ((k ^ (r & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[4 * kk]), "r"(pk[4 * kk + 1]),
                     "r"(pk[4 * kk + 2]), "r"(pk[4 * kk + 3])
                     : "memory");
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(1 + x, TILE_THREADS);
    if (lead && ok) {
      if constexpr (C::PACKED)
        tma_store_5d(tmO, stage0 + buf * C::CHUNK_BYTES, 64 * c64, 0, hkv, t.tok0, b);
      else
        tma_store_4d(tmO, stage0 + buf * C::CHUNK_BYTES, 64 * c64, t.h, t.q0, b);
      bulk_commit();
    }
  }
  const float lse = l > 0.f ? (m + __log2f(l) - log2g) * 0.69314718055994531f : -INFINITY;
  if (C::PACKED && p.n_parts > 1) {
    if (row < p.Sq && ok) p.lse_part[(((int64_t)t.part * p.B + b) * p.Hq + head) * p.Sq + row] = lse;
  } else if (p.lse != nullptr && row < p.Sq && ok) {
    p.lse[bhq * p.Sq + row] = lse;
  }
  if (lead) bulk_wait0();
}


// ------------------------------------------------------------------ kernel --
template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ AttnParams p, const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmO) {
  using namespace ptx;
  // Decode: the split merge that follows may be launched now (it waits for
  // this grid's completion itself); every CTA of this grid is resident by then.
  if constexpr (C::PACKED) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // Q buffers, then E4M3 P buffers (shared-memory P), then the K/V ring. With one
  // query tile per CTA the second tile's pointers alias the first (never used).
  uint8_t* const sQ[2] = {smem, smem + (C::NQ - 1) * C::Q_TILE};
  uint8_t* const sP[2] = {smem + C::NQ * C::Q_TILE, smem + C::NQ * C::Q_TILE + C::P_BYTES / 2};
  uint8_t* sSlots = smem + C::NQ * C::Q_TILE + C::P_BYTES;  // the K/V ring (split: K ring, then V ring)
  AttnMisc* misc = reinterpret_cast<AttnMisc*>(sSlots + C::RING_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item -> (b, heads, query rows) ----
  int b, hkv;
  TileInfo t[2];
  if constexpr (C::PACKED) {
    // (unit pair, split, kv head, batch); rows are Sq * group packed rows.
    int item = blockIdx.x;
    const int pr = item % p.n_units;
    item /= p.n_units;
    const int split = item % p.n_splits;
    item /= p.n_splits;
    hkv = item % p.Hkv;
    b = item / p.Hkv;
    const int toks = C::BM >> p.group_shift;  // query tokens per 128-row unit
    for (int x = 0; x < 2; ++x) {
      t[x].h = hkv * p.group;
      t[x].qblk = p.kv_interleave ? 0 : 2 * pr + x;  // interleaved: both tiles hold all rows
      t[x].q0 = t[x].qblk * C::BM;
      t[x].tok0 = t[x].qblk * toks;
      t[x].mrow = t[x].tok0 / C::BM;
      t[x].valid = t[x].q0 < p.n_rows;
      int n = p.n_kv_blocks;  // causal / length limit; the split's tiles are chosen below
      if (p.causal) {
        const int last = min(t[x].tok0 + toks - 1, p.Sq - 1) + (p.Skv - p.Sq);
        n = last < 0 ? 0 : min(p.n_kv_blocks, last / C::BN + 1);
      }
      t[x].n_kv = t[x].valid ? n : 0;
      t[x].u0 = 0;
      t[x].x = x;
      t[x].part = p.kv_interleave ? 2 * split + x : split;
    }
    // Warp 2 (idle) picks the split's kept KV tiles: rank r of the kept tiles
    // in [0, n) goes to split r / per; interleaved tiles take alternate ranks.
    if (warp == 2) {
      // Words past the larger tile's limit are never read; those below it are
      // all written (shared memory starts with stale contents).
      const int n_words = (max(t[0].n_kv, t[1].n_kv) + 31) >> 5;
      for (int x = 0; x < 2; ++x) {
        if (p.kv_interleave && x == 1) break;  // tile 1 shares tile 0's scan
        const int n = t[x].n_kv;
        const uint8_t* mrow = p.mask == nullptr ? nullptr
                              : p.mask + b * p.mask_sb + hkv * p.mask_sh + static_cast<int64_t>(t[x].mrow) * p.n_kv_blocks;
        int total = 0;
        for (int base = 0; base < n; base += 32) {
          const int u = base + lane;
          const bool k = u < n && (mrow == nullptr || mrow[u] != 0);
          total += __popc(__ballot_sync(0xffffffffu, k));
        }
        const int per = (total + p.n_splits - 1) / p.n_splits;
        const int r0 = split * per, r1 = min(total, r0 + per);
        int lo[2] = {1 << 30, 1 << 30}, hi[2] = {0, 0};
        int cnt = 0;
        for (int base = 0; base < (n_words << 5); base += 32) {
          const int u = base + lane;
          const bool k = u < n && (mrow == nullptr || mrow[u] != 0);
          const uint32_t bal = __ballot_sync(0xffffffffu, k);
          const int rank = cnt + __popc(bal & ((1u << lane) - 1u));
          const bool mine = k && rank >= r0 && rank < r1;
          const int dest = p.kv_interleave ? ((rank - r0) & 1) : x;
          const uint32_t b0 = __ballot_sync(0xffffffffu, mine && dest == 0);
          const uint32_t b1 = __ballot_sync(0xffffffffu, mine && dest == 1);
          if (lane == 0) {
            if (p.kv_interleave) {
              misc->keep_bits[0][base >> 5] = b0;
              misc->keep_bits[1][base >> 5] = b1;
            } else {
              misc->keep_bits[x][base >> 5] = x ? b1 : b0;
            }
          }
          if (b0) { lo[0] = min(lo[0], base + __ffs(b0) - 1); hi[0] = base + 32 - __clz(b0); }
          if (b1) { lo[1] = min(lo[1], base + __ffs(b1) - 1); hi[1] = base + 32 - __clz(b1); }
          cnt += __popc(bal);
        }
        if (lane == 0) {
          if (p.kv_interleave) {
            for (int y = 0; y < 2; ++y) { misc->range[y][0] = lo[y]; misc->range[y][1] = hi[y]; }
          } else {
            misc->range[x][0] = lo[x];
            misc->range[x][1] = hi[x];
          }
        }
      }
    }
  } else {
    int item = blockIdx.x;
    if (C::SPLIT) {  // SINGLE: one query block of one head, its kept KV tiles split between the warpgroups
      int qb = item % p.n_units;
      item /= p.n_units;
      const int h = item % p.Hq;
      b = item / p.Hq;
      if (p.causal) qb = p.n_units - 1 - qb;  // heaviest causal tiles first
      t[0].h = t[1].h = h;
      t[0].qblk = t[1].qblk = qb;
    } else if (p.pair_mode == PAIR_ROWS) {
      int pr = item % p.n_units;
      item /= p.n_units;
      const int h = item % p.Hq;
      b = item / p.Hq;
      if (p.causal) pr = p.n_units - 1 - pr;  // heaviest causal tiles first
      for (int x = 0; x < 2; ++x) {
        t[x].h = h;
        t[x].qblk = 2 * pr + x;
      }
    } else {
      int qb = item % p.n_units;
      item /= p.n_units;
      const int hp = item % (p.Hq / 2);
      b = item / (p.Hq / 2);
      if (p.causal) qb = p.n_units - 1 - qb;
      for (int x = 0; x < 2; ++x) {
        t[x].h = 2 * hp + x;
        t[x].qblk = qb;
      }
    }
    hkv = t[0].h / p.group;
    for (int x = 0; x < 2; ++x) {
      t[x].q0 = t[x].qblk * C::BM;
      t[x].tok0 = t[x].q0;
      t[x].mrow = t[x].qblk;
      t[x].u0 = 0;
      t[x].x = x;
      t[x].part = 0;
      t[x].valid = t[x].q0 < p.Sq;
      int n = p.n_kv_blocks;
      if (p.causal) {
        const int last = min(t[x].q0 + C::BM - 1, p.Sq - 1) + (p.Skv - p.Sq);
        n = last < 0 ? 0 : min(p.n_kv_blocks, last / C::BN + 1);
      }
      t[x].n_kv = t[x].valid ? n : 0;
    }
    // Split tiles: warp 2 gives the kept KV tiles (causal bound, block mask) of
    // the query tile alternately to the two warpgroups: ranks 0, 2, 4, ... to
    // warpgroup 0 and 1, 3, 5, ... to warpgroup 1. same_kept holds the number
    // of tiles both have (exp turn-taking runs over those).
    if (C::SPLIT && warp == 2) {
      const int n_words = (t[0].n_kv + 31) >> 5;
      const uint8_t* mrow = p.mask == nullptr ? nullptr
                            : p.mask + b * p.mask_sb + hkv * p.mask_sh + static_cast<int64_t>(t[0].mrow) * p.n_kv_blocks;
      int total = 0;
      for (int wd = 0; wd < n_words; ++wd) {
        const int u = (wd << 5) + lane;
        const bool kept = u < t[0].n_kv && (mrow == nullptr || mrow[u] != 0);
        const uint32_t kb = __ballot_sync(0xffffffffu, kept);
        const int rank = total + __popc(kb & ((1u << lane) - 1u));
        const uint32_t even = __ballot_sync(0xffffffffu, kept && (rank & 1) == 0);
        if (lane == 0) {
          misc->keep_bits[0][wd] = even;
          misc->keep_bits[1][wd] = kb & ~even;
        }
        total += __popc(kb);
      }
      if (lane == 0) misc->same_kept = total >> 1;
    }
    // Masked launch: warp 2 (otherwise idle) turns each query tile's block-mask
    // row into the keep-bit set (one coalesced 32-byte read per word), and
    // records whether both tiles keep the same KV tiles.
    if (!C::SPLIT && p.mask != nullptr && warp == 2) {
      const int n_words = (max(t[0].n_kv, t[1].n_kv) + 31) >> 5;
      bool same = t[0].n_kv == t[1].n_kv;
      int count = 0;
      for (int wd = 0; wd < n_words; ++wd) {
        uint32_t bits[2];
        for (int x = 0; x < 2; ++x) {
          const uint8_t* mrow =
              p.mask + b * p.mask_sb + hkv * p.mask_sh + static_cast<int64_t>(t[x].mrow) * p.n_kv_blocks;
          const int u = (wd << 5) + lane;
          bits[x] = __ballot_sync(0xffffffffu, u < t[x].n_kv && mrow[u] != 0);
          if (lane == 0) misc->keep_bits[x][wd] = bits[x];
        }
        same = same && bits[0] == bits[1];
        count += __popc(bits[0]);
      }
      if (lane == 0) misc->same_kept = same ? count : 0;
    }
  }

  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&misc->q_full), 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(smem_addr(&misc->s_full[x]), 1);
      mbar_init(smem_addr(&misc->p_full[x]), 4);  // one arrive per softmax warp
    }
    mbar_init(smem_addr(&misc->o_full), 1);
    mbar_init(smem_addr(&misc->drain), 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(smem_addr(&misc->s_free[x]), 4);  // one arrive per softmax warp
      mbar_init(smem_addr(&misc->pv_done[x]), 1);
      mbar_init(smem_addr(&misc->exp_done[x]), 4);  // one arrive per softmax warp
    }
    for (int s = 0; s < (C::SPLIT ? C::K_STAGES + C::V_STAGES : C::STAGES); ++s) {
      mbar_init(smem_addr(&misc->kv_full[s]), 1);
      mbar_init(smem_addr(&misc->kv_empty[s]), 1);
    }
    misc->abort = 0u;
    fence_barrier_init();
  }
  if (C::PV == PV_E4M3 && p.sf_v_kind == FMHA_SF_PER_CHANNEL && threadIdx.x < C::DV)
    misc->sf_v[threadIdx.x] = p.sf_v[(static_cast<int64_t>(b) * p.Hkv + hkv) * C::DV + threadIdx.x];
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_addr(&misc->tmem_base), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == C::LOAD_WARP && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc->tmem_base;
  const Waiter w{&misc->abort, p.err, p.wait_cycles};
  if constexpr (C::PACKED) {
    for (int x = 0; x < 2; ++x) {
      if (t[x].valid) {
        t[x].u0 = misc->range[x][0];
        t[x].n_kv = misc->range[x][1];
      } else {
        t[x].u0 = 1 << 30;
        t[x].n_kv = 0;
      }
    }
  }

  if (warp >= C::SOFTMAX_WARP0) {
    regs_inc<C::SOFTMAX_REGS>();
    const int x = (warp - C::SOFTMAX_WARP0) >> 2;  // query tile
    const TileInfo tx = x ? t[1] : t[0];  // select by value (no runtime-indexed array)
    // Exp turn-taking needs both tiles to walk the same KV tiles: without a
    // mask their common prefix [0, min n_kv); with a block mask only when both
    // tiles keep the same tiles (e.g. two query heads of one KV head).
    int n_turns = 0;
    if (C::TURNS && !C::PACKED)
      n_turns = (C::SPLIT || p.mask != nullptr) ? misc->same_kept : min(t[0].n_kv, t[1].n_kv);
    if (tx.valid)
      attn_softmax_role<C>(p, tx, x, b, hkv, x ? sQ[1] : sQ[0], x ? sP[1] : sP[0], sSlots, n_turns, misc, tmem,
                           &tmO, w);
  } else {
    regs_dec<C::CONTROL_REGS>();
    uint8_t* const sV = sSlots + C::K_STAGES * C::K_TILE;  // split: the V ring
    if (warp == C::MMA_WARP) {  // the whole warp; one elected lane issues
      if constexpr (C::SPLIT && C::PSMEM)
        attn_mma_role_psmem_split<C>(p, t[0], sQ[0], sP[0], sP[1], sSlots, sV, misc, tmem, w);
      else if constexpr (C::SPLIT)
        attn_mma_role_split<C>(p, t[0], t[1], sQ[0], sSlots, sV, misc, tmem, w);
      else if constexpr (C::PSMEM)
        attn_mma_role_psmem<C>(p, t[0], t[1], b, hkv, sQ[0], sQ[1], sP[0], sP[1], sSlots, misc, tmem, w);
      else
        attn_mma_role<C>(p, t[0], t[1], b, hkv, sQ[0], sQ[1], sSlots, misc, tmem, w);
    } else if (C::SPLIT && (warp == C::LOAD_WARP || warp == C::LOAD_WARP + 2)) {
      // split tiles: warp 1 loads Q and the K ring, warp 3 the V ring
      attn_load_role_split<C>(p, t[0], b, hkv, warp == C::LOAD_WARP ? 0 : 1, sQ[0], sSlots, sV, misc, &tmQ,
                              &tmK, &tmV, w);
    } else if (warp == C::LOAD_WARP) {  // the whole warp
      attn_load_role<C>(p, t[0], t[1], b, hkv, sQ[0], sQ[1], sSlots, misc, &tmQ, &tmK, &tmV, w);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <class C>
cudaError_t launch_attention_t(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const CUtensorMap& to, cudaStream_t stream) {
  auto kern = attn_fwd_kernel<C>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int head_units = C::PACKED ? p.Hkv * p.n_splits : (p.pair_mode == PAIR_HEADS ? p.Hq / 2 : p.Hq);
  const long long blocks = static_cast<long long>(p.n_units) * head_units * p.B;
  kern<<<static_cast<unsigned>(blocks), C::THREADS, C::SMEM_BYTES, stream>>>(p, tq, tk, tv, to);
  return cudaGetLastError();
}

// The two-term-P and E4M3-output variants of one (D, QK, PV, PAGED) kernel.
template <int D, int QK, int PV, bool PAGED>
cudaError_t launch_attention_variants(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                                      const CUtensorMap& tv, const CUtensorMap& to, cudaStream_t s) {
  static_assert(D == 64 || D == 128, "the 192-wide QK kernels have their own instantiation unit");
  if constexpr (PV == PV_E4M3) {
    if (p.p_terms == 2)
      return p.o8 ? launch_attention_t<AttnCfg<D, QK, PV, PAGED, true, false, true>>(p, tq, tk, tv, to, s)
                  : launch_attention_t<AttnCfg<D, QK, PV, PAGED, true>>(p, tq, tk, tv, to, s);
  }
  if constexpr (D == 128) {
    if (p.o8) return launch_attention_t<AttnCfg<D, QK, PV, PAGED, false, false, true>>(p, tq, tk, tv, to, s);
  }
  return launch_attention_t<AttnCfg<D, QK, PV, PAGED>>(p, tq, tk, tv, to, s);
}

}  // namespace fmha
