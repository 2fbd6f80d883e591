// Warp-specialised tcgen05 tile engine shared by every tensor-core kernel of
// the library.
//
// One CTA per SM (persistent), 192 threads:
//   warp 0      one thread issues TMA tile loads into a STAGES-deep ring of
//               shared-memory stages (A: 128 x 64 bf16, B: 256 x 64 bf16);
//   warp 1      allocates 512 TMEM columns; one thread issues
//               tcgen05.mma (M=128, N=256, K=16) into one of two 256-column
//               fp32 accumulators, so the epilogue of tile t overlaps the
//               MMAs of tile t+1;
//   warps 2..5  the epilogue: thread (warp&3)*32+lane owns accumulator row
//               (TMEM lane) (warp&3)*32+lane and reads it with tcgen05.ld.
// A policy class supplies the tile order (identical for all roles), the TMA
// coordinates and the epilogue.  Operands may be K-major (rows of K) or
// MN-major (rows of M/N) in global memory; both are staged with 128-byte
// swizzling, which the UMMA descriptors describe.
#pragma once

#include <type_traits>
#include <utility>

#include "cce_ptx.cuh"

namespace cce {

constexpr int BM = 128;   // accumulator rows (TMEM lanes)
constexpr int BN = 256;   // accumulator columns
constexpr int BK = 64;    // K per stage: one 128-byte swizzle row of bf16
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr int EPI_THREADS = 128;
constexpr uint32_t TMEM_COLS = 512;

struct Ctl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int consumed;
  int pad;
  // Stage records of the masked path, written by the producer before it
  // arrives on full[s] and read by the MMA issuer after waiting on it:
  // bits 0..3 = K=16 steps to issue, REC_LAST = last stage of its tile.
  uint32_t rec[STAGES];
};
constexpr uint32_t REC_LAST = 1u << 4;

// Dynamic shared memory of a policy's kernel: the stage ring, the policy's
// own 1024-aligned epilogue buffer (Policy::EXTRA_SMEM bytes) and the control
// block, plus alignment slack.
template <class Policy>
constexpr int smem_bytes() {
  return STAGES * STAGE_BYTES + Policy::EXTRA_SMEM + static_cast<int>(sizeof(Ctl)) + 1024 + 64;
}

struct Pipe {
  int stage = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void advance() {
    if (++stage == STAGES) {
      stage = 0;
      phase ^= 1u;
    }
  }
};

// Sequential reader of a K-step mask: bit (kb & 7) * 4 + kk of word kb >> 3
// is set when the K=16 step kk of stage kb must be issued.  The next word is
// fetched one word ahead so the single MMA-issuing thread rarely waits on it.
// A null mask means every step is issued.
struct MaskCursor {
  const uint32_t* p;
  uint32_t cur, nxt;
  int nwords;
  __device__ __forceinline__ void init(const uint32_t* m, int nkb) {
    p = m;
    nwords = (nkb + 7) >> 3;
    cur = (m && nwords > 0) ? __ldg(m) : 0xFFFFFFFFu;
    nxt = (m && nwords > 1) ? __ldg(m + 1) : 0u;
  }
  // must be called for kb = 0, 1, 2, ... in order
  __device__ __forceinline__ uint32_t bits(int kb) {
    if (!p) return 0xFu;
    if (kb > 0 && (kb & 7) == 0) {
      cur = nxt;
      const int w = (kb >> 3) + 1;
      nxt = w < nwords ? __ldg(p + w) : 0u;
    }
    return (cur >> ((kb & 7) * 4)) & 0xFu;
  }
};

// ---------------------------------------------------------------------------
// Order of (row block, inner index) work items that keeps the row operand
// resident in L2.  Every item re-reads its 128-row block of H (the A operand,
// K = D) from L2 once per vocabulary tile; if all row blocks were live at once
// (inner-major order), their blocks together (N x D x 2 bytes, 134 MB at
// N = 16384, D = 4096) would exceed L2 and every re-read would go to DRAM.
// Instead the row blocks are taken in groups whose bytes stay below
// kRowGroupBytes; within a group the inner index (vocabulary split or tile)
// is the major one, so the CTAs running at the same time share each vocabulary
// tile and keep re-reading the same group of row blocks.  E is then read from
// DRAM once per group.
#ifndef CCE_ROW_GROUP_MB
#define CCE_ROW_GROUP_MB 40
#endif
constexpr long long kRowGroupBytes = (long long)CCE_ROW_GROUP_MB << 20;

// Row blocks per group for num_mb blocks of blk_bytes each: as few groups as
// the budget allows, of near-equal size.
__device__ __forceinline__ int row_group_blocks(int num_mb, long long blk_bytes) {
  const long long total = (long long)num_mb * blk_bytes;
  const int ngroups = (int)max(1ll, (total + kRowGroupBytes - 1) / kRowGroupBytes);
  return max(1, (num_mb + ngroups - 1) / ngroups);
}

// Item -> (row block, inner index) for items 0 .. num_mb * n_inner - 1, in
// groups of gm row blocks (the last group may be smaller).
__device__ __forceinline__ void grouped_item(int item, int num_mb, int n_inner, int gm, int& mb,
                                             int& inner) {
  const int full = num_mb / gm;  // complete groups
  const int per = gm * n_inner;  // items per complete group
  const int g = item / per;
  if (g < full) {
    const int r = item - g * per;
    inner = r / gm;
    mb = g * gm + (r - inner * gm);
  } else {
    const int rem = num_mb - full * gm;  // > 0 here
    const int r = item - full * per;
    inner = r / rem;
    mb = full * gm + (r - inner * rem);
  }
}

// Index of the last stage of a K-step mask (see MaskCursor) with any step to
// issue, among stages 0 .. nkb-1; -1 if none; nkb - 1 for a null mask.
__device__ __forceinline__ int mask_last_stage(const uint32_t* m, int nkb) {
  if (!m) return nkb - 1;
  const int nwords = (nkb + 7) >> 3;
  for (int w = nwords - 1; w >= 0; --w) {
    uint32_t v = __ldg(m + w);
    const int stages = min(8, nkb - w * 8);
    if (stages < 8) v &= (1u << (stages * 4)) - 1u;
    if (v) return w * 8 + ((31 - __clz(v)) >> 2);
  }
  return -1;
}

// Per-role state handed to policies.
struct Engine {
  Ctl* ctl;
  uint8_t* smem;   // 1024-byte aligned stage ring
  uint8_t* extra;  // 1024-byte aligned policy epilogue buffer
  uint32_t tmem;
  int* status;
  Pipe pipe;
  int tcount = 0;  // accumulator tiles handled by this role
  int fills = 0;   // stage fills issued (producer) / consumed (MMA)
  uint64_t wait_ns = kWaitLimitNs;  // limit of every wait of this launch

  __device__ __forceinline__ volatile int* abort_flag() { return &ctl->abort; }
  // Bounded wait on a barrier phase (see wait_parity).
  __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity) {
    return wait_parity(bar, parity, abort_flag(), status, wait_ns);
  }

  // ---- producer: load nkb stages of one tile.  (ax, ay) / (bx, by) are the
  // tensor-map coordinates of the tile origin; K advances along x for a
  // K-major operand and along y for an MN-major one.  With a K-step mask
  // (see mma()), stages whose four K=16 steps are all masked are not loaded.
  template <bool A_MN, bool B_MN>
  __device__ __forceinline__ bool produce(const CUtensorMap* mA, const CUtensorMap* mB, int ax,
                                          int ay, int bx, int by, int nkb,
                                          const uint32_t* kmask = nullptr) {
    MaskCursor mc;
    mc.init(kmask, nkb);
    for (int kb = 0; kb < nkb; ++kb) {
      if (!mc.bits(kb)) continue;
      if (!wait(smem_u32(&ctl->empty[pipe.stage]), pipe.phase ^ 1u))
        return false;
      const uint32_t fb = smem_u32(&ctl->full[pipe.stage]);
      mbar_arrive_expect_tx(fb, STAGE_BYTES);
      const uint32_t sa = smem_u32(smem + pipe.stage * STAGE_BYTES);
      const uint32_t sb = sa + A_BYTES;
      if (!A_MN) {
        tma_load_2d(sa, mA, fb, ax + kb * BK, ay);
      } else {
        tma_load_2d(sa, mA, fb, ax, ay + kb * BK);
        tma_load_2d(sa + 8192, mA, fb, ax + 64, ay + kb * BK);
      }
      if (!B_MN) {
        tma_load_2d(sb, mB, fb, bx + kb * BK, by);
      } else {
#pragma unroll
        for (int b = 0; b < 4; ++b) tma_load_2d(sb + b * 8192, mB, fb, bx + b * 64, by + kb * BK);
      }
      pipe.advance();
      ++fills;
    }
    return true;
  }

  // ---- MMA issuer: accumulate one tile over nkb stages into the next
  // accumulator.  kmask (optional) has bit kb*4+kk set for every K=16 step
  // that must be issued; cleared bits are skipped (all-zero A slices).  When
  // a mask skips every step the accumulator is left untouched, so the
  // policy's epilogue must recognise such a tile from the same mask and
  // treat it as zero.
  template <bool A_MN, bool B_MN>
  __device__ __forceinline__ bool mma(int nkb, const uint32_t* kmask = nullptr) {
    const int acc = tcount & 1;
    if (!wait(smem_u32(&ctl->tempty[acc]), (((uint32_t)tcount >> 1) & 1u) ^ 1u))
      return false;
    tc_fence_after();
    const uint32_t d = tmem + acc * BN;
    constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, A_MN, B_MN);
    uint32_t issued = 0;
    MaskCursor mc;
    mc.init(kmask, nkb);
    for (int kb = 0; kb < nkb; ++kb) {
      const uint32_t bits = mc.bits(kb);
      if (!bits) continue;  // the producer skipped this stage too
      if (!wait(smem_u32(&ctl->full[pipe.stage]), pipe.phase))
        return false;
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + pipe.stage * STAGE_BYTES);
      const uint32_t sb = sa + A_BYTES;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        if (!(bits & (1u << kk))) continue;
        const uint64_t ad = A_MN ? smem_desc_sw128(sa + kk * 2048, 8192, 1024)
                                 : smem_desc_sw128(sa + kk * 32, 16, 1024);
        const uint64_t bd = B_MN ? smem_desc_sw128(sb + kk * 2048, 8192, 1024)
                                 : smem_desc_sw128(sb + kk * 32, 16, 1024);
        umma_bf16(d, ad, bd, idesc, issued);
        issued = 1;
      }
      umma_commit(smem_u32(&ctl->empty[pipe.stage]));
      pipe.advance();
      ++fills;
    }
    umma_commit(smem_u32(&ctl->tfull[acc]));
    ++tcount;
    return true;
  }

  // ---- masked producer (lane 0): like produce() with a K-step mask, but the
  // MMA issuer never reads the mask: each loaded stage carries a record (its
  // non-zero K steps, and REC_LAST on the tile's last loaded stage, found by
  // scanning the mask first), written before the stage is announced.  A tile
  // with no non-zero stage still sends one empty REC_LAST stage.
  template <bool A_MN, bool B_MN>
  __device__ __forceinline__ bool produce_rec(const CUtensorMap* mA, const CUtensorMap* mB, int ax,
                                              int ay, int bx, int by, int nkb,
                                              const uint32_t* kmask) {
    const int last = mask_last_stage(kmask, nkb);
    if (last < 0) {  // nothing to load: one empty stage ends the tile
      if (!wait(smem_u32(&ctl->empty[pipe.stage]), pipe.phase ^ 1u)) return false;
      ctl->rec[pipe.stage] = REC_LAST;
      mbar_arrive(smem_u32(&ctl->full[pipe.stage]));
      pipe.advance();
      ++fills;
      return true;
    }
    MaskCursor mc;
    mc.init(kmask, nkb);
    for (int kb = 0; kb <= last; ++kb) {
      const uint32_t bits = mc.bits(kb);
      if (!bits) continue;
      if (!wait(smem_u32(&ctl->empty[pipe.stage]), pipe.phase ^ 1u))
        return false;
      const uint32_t fb = smem_u32(&ctl->full[pipe.stage]);
      ctl->rec[pipe.stage] = bits | (kb == last ? REC_LAST : 0u);
      mbar_arrive_expect_tx(fb, STAGE_BYTES);
      const uint32_t sa = smem_u32(smem + pipe.stage * STAGE_BYTES);
      const uint32_t sb = sa + A_BYTES;
      if (!A_MN) {
        tma_load_2d(sa, mA, fb, ax + kb * BK, ay);
      } else {
        tma_load_2d(sa, mA, fb, ax, ay + kb * BK);
        tma_load_2d(sa + 8192, mA, fb, ax + 64, ay + kb * BK);
      }
      if (!B_MN) {
        tma_load_2d(sb, mB, fb, bx + kb * BK, by);
      } else {
#pragma unroll
        for (int b = 0; b < 4; ++b) tma_load_2d(sb + b * 8192, mB, fb, bx + b * 64, by + kb * BK);
      }
      pipe.advance();
      ++fills;
    }
    return true;
  }

  // ---- masked MMA issuer: consumes the producer's records until REC_LAST.
  template <bool A_MN, bool B_MN>
  __device__ __forceinline__ bool mma_rec() {
    const int acc = tcount & 1;
    if (!wait(smem_u32(&ctl->tempty[acc]), (((uint32_t)tcount >> 1) & 1u) ^ 1u))
      return false;
    tc_fence_after();
    const uint32_t d = tmem + acc * BN;
    constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, A_MN, B_MN);
    constexpr uint32_t a_step = A_MN ? 2048 : 32;  // bytes per K=16 step
    constexpr uint32_t b_step = B_MN ? 2048 : 32;
    const uint64_t ad0 = A_MN ? smem_desc_sw128(smem_u32(smem), 8192, 1024)
                              : smem_desc_sw128(smem_u32(smem), 16, 1024);
    const uint64_t bd0 = B_MN ? smem_desc_sw128(smem_u32(smem) + A_BYTES, 8192, 1024)
                              : smem_desc_sw128(smem_u32(smem) + A_BYTES, 16, 1024);
    uint32_t issued = 0;
    for (;;) {
      if (!wait(smem_u32(&ctl->full[pipe.stage]), pipe.phase))
        return false;
      const uint32_t rec = *reinterpret_cast<volatile uint32_t*>(&ctl->rec[pipe.stage]);
      const uint64_t so = (uint64_t)((pipe.stage * STAGE_BYTES) >> 4);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        if (!(rec & (1u << kk))) continue;
        umma_bf16(d, ad0 + so + kk * (a_step >> 4), bd0 + so + kk * (b_step >> 4), idesc, issued);
        issued = 1;
      }
      umma_commit(smem_u32(&ctl->empty[pipe.stage]));
      pipe.advance();
      ++fills;
      if (rec & REC_LAST) break;
    }
    umma_commit(smem_u32(&ctl->tfull[acc]));
    ++tcount;
    return true;
  }

  // ---- epilogue: wait for the next accumulator; returns its TMEM address
  // for this thread's lane quarter (column 0).
  __device__ __forceinline__ bool epi_acquire(int quarter, uint32_t& taddr) {
    const int acc = tcount & 1;
    if (!wait(smem_u32(&ctl->tfull[acc]), ((uint32_t)tcount >> 1) & 1u))
      return false;
    tc_fence_after();
    taddr = tmem + acc * BN + ((uint32_t)(quarter * 32) << 16);
    return true;
  }
  __device__ __forceinline__ void epi_release(int lane) {
    const int acc = tcount & 1;
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&ctl->tempty[acc]));
    ++tcount;
  }
  // ---- epilogue over a pair of tiles (t, t+1) held at once, one in each
  // accumulator (used when a work unit computes two products of the same
  // shape, e.g. teacher and student logits).  The MMA of the next pair waits
  // until both are released, so the pair's epilogue does not overlap it.
  __device__ __forceinline__ bool epi_acquire2(int quarter, uint32_t& ta, uint32_t& tb) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int t = tcount + k;
      if (!wait(smem_u32(&ctl->tfull[t & 1]), ((uint32_t)t >> 1) & 1u))
        return false;
    }
    tc_fence_after();
    const uint32_t lanes = (uint32_t)(quarter * 32) << 16;
    ta = tmem + (tcount & 1) * BN + lanes;
    tb = tmem + ((tcount + 1) & 1) * BN + lanes;
    return true;
  }
  __device__ __forceinline__ void epi_release2(int lane) {
    epi_release(lane);
    epi_release(lane);
  }
};

// ===========================================================================
// CTA-pair engine (tcgen05 cta_group::2).  A cluster of two CTAs computes one
// 256 x 256 accumulator tile: each CTA stages its own 128 rows of A and 128 of
// B's 256 columns per K step (32 KiB stages, PAIR_STAGES deep), the rank-0
// CTA's single MMA thread issues M = 256 MMAs that read both CTAs' shared
// memory, and each CTA's tensor memory holds its own 128 accumulator rows
// (two 256-column accumulators, so the epilogue of a tile overlaps the MMAs of
// the next).  Compared with one CTA per 128 x 256 tile, every CTA moves a
// third fewer operand bytes per FLOP from L2 and keeps 1.5x more bytes in
// flight.
//   Barriers: full[s] lives in the rank-0 CTA (one arrival, by its producer,
//   with the bytes of both CTAs' copies, which complete on it); empty[s] and
//   tfull[a] live in both CTAs and are signalled by the MMA thread's commits
//   (one commit arrives on the same barrier in both CTAs);
//   tempty[a] lives in the rank-0 CTA and receives the arrivals of both CTAs'
//   epilogue warps.  Every wait is bounded (wait_parity).
// ===========================================================================
constexpr int PAIR_STAGES = 6;
constexpr int PA_BYTES = 128 * BK * 2;  // this CTA's A rows of one stage
constexpr int PB_BYTES = 128 * BK * 2;  // this CTA's half of B's columns
constexpr int PSTAGE_BYTES = PA_BYTES + PB_BYTES;
// Dual-product stages (PairEngineT::produce_dual): two A operands of 128 rows
// and this CTA's 64 rows of a 128-row B operand, 40 KiB, five deep.
constexpr int PAIR_DUAL_STAGES = 5;
constexpr int PDUAL_STAGE_BYTES = 2 * PA_BYTES + 64 * BK * 2;

template <int NST>
struct PairCtlT {
  uint64_t full[NST];
  uint64_t empty[NST];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int consumed;
  int pad;
  uint32_t rec[NST];
};

// Stage geometry of a pair policy: Policy::PAIR_NST stages of
// Policy::PAIR_SB bytes when it declares them, else the 32 KiB default.
template <class P, class = void>
struct PairGeom {
  static constexpr int NST = PAIR_STAGES;
  static constexpr int SB = PSTAGE_BYTES;
};
template <class P>
struct PairGeom<P, std::void_t<decltype(P::PAIR_NST), decltype(P::PAIR_SB)>> {
  static constexpr int NST = P::PAIR_NST;
  static constexpr int SB = P::PAIR_SB;
};

template <class Policy>
constexpr int pair_smem_bytes() {
  using G = PairGeom<Policy>;
  return G::NST * G::SB + Policy::EXTRA_SMEM + static_cast<int>(sizeof(PairCtlT<G::NST>)) + 1024 +
         64;
}

template <int NST>
struct PairPipe {
  int stage = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void advance() {
    if (++stage == NST) {
      stage = 0;
      phase ^= 1u;
    }
  }
};

// K-step bits of stage kb in the union of two masks (see MaskCursor); a null
// mask issues every step.
struct MaskPair {
  MaskCursor a, b;
  bool any_null;
  __device__ __forceinline__ void init(const uint32_t* m0, const uint32_t* m1, int nkb) {
    any_null = (m0 == nullptr) || (m1 == nullptr);
    a.init(m0, nkb);
    b.init(m1, nkb);
  }
  __device__ __forceinline__ uint32_t bits(int kb) {
    const uint32_t x = a.bits(kb), y = b.bits(kb);
    return any_null ? 0xFu : (x | y);
  }
};

template <int NST, int SB>
struct PairEngineT {
  PairCtlT<NST>* ctl;
  uint8_t* smem;
  uint8_t* extra;
  uint32_t tmem;
  int* status;
  uint32_t rank;  // 0: issues the MMAs; 1: its peer
  PairPipe<NST> pipe;
  int tcount = 0;
  int fills = 0;
  uint64_t wait_ns = kWaitLimitNs;

  __device__ __forceinline__ volatile int* abort_flag() { return &ctl->abort; }
  __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity) {
    return wait_parity(bar, parity, abort_flag(), status, wait_ns);
  }
  // shared::cluster address of a barrier of this CTA's layout in CTA `r`
  __device__ __forceinline__ uint32_t in_cta(const uint64_t* bar, uint32_t r) const {
    return mapa_shared(smem_u32(bar), r);
  }

  // ---- producer (each CTA, lane 0 of warp 0): this CTA's halves of one
  // tile's stages.  (ax, ay) / (bx, by) are the tensor-map coordinates of this
  // CTA's A rows and B columns; K advances along x for a K-major operand, y
  // for an MN-major one.  Stages whose K steps are zero in both CTAs' masks
  // are skipped by both; each loaded stage carries a record for the MMA
  // thread (its K steps, REC_LAST on the tile's last stage, found by scanning
  // both masks first), written by the rank-0 producer before it announces
  // the stage with the bytes of both CTAs' copies.
  template <bool A_MN, bool B_MN>
  __device__ __forceinline__ bool produce_rec(const CUtensorMap* mA, const CUtensorMap* mB, int ax,
                                              int ay, int bx, int by, int nkb, const uint32_t* m0,
                                              const uint32_t* m1) {
    constexpr uint32_t tx = 2u * SB;
    const int last = (m0 == nullptr || m1 == nullptr)
                         ? nkb - 1
                         : max(mask_last_stage(m0, nkb), mask_last_stage(m1, nkb));
    if (last < 0) {  // nothing to load: one empty stage ends the tile (both CTAs keep step)
      if (!wait(smem_u32(&ctl->empty[pipe.stage]), pipe.phase ^ 1u)) return false;
      if (rank == 0) {
        ctl->rec[pipe.stage] = REC_LAST;
        mbar_arrive(smem_u32(&ctl->full[pipe.stage]));
      }
      pipe.advance();
      ++fills;
      return true;
    }
    MaskPair mc;
    mc.init(m0, m1, nkb);
    for (int kb = 0; kb <= last; ++kb) {
      const uint32_t bits = mc.bits(kb);
      if (!bits) continue;
      if (!wait(smem_u32(&ctl->empty[pipe.stage]), pipe.phase ^ 1u)) return false;
      if (rank == 0) {
        ctl->rec[pipe.stage] = bits | (kb == last ? REC_LAST : 0u);
        mbar_arrive_expect_tx(smem_u32(&ctl->full[pipe.stage]), tx);
      }
      const uint32_t fb = in_cta(&ctl->full[pipe.stage], 0);
      const uint32_t sa = smem_u32(smem + pipe.stage * SB);
      const uint32_t sb = sa + PA_BYTES;
      if (!A_MN) {
        tma_load_2d_pair(sa, mA, fb, ax + kb * BK, ay);
      } else {
        tma_load_2d_pair(sa, mA, fb, ax, ay + kb * BK);
        tma_load_2d_pair(sa + 8192, mA, fb, ax + 64, ay + kb * BK);
      }
      if (!B_MN) {
        tma_load_2d_pair(sb, mB, fb, bx + kb * BK, by);
      } else {
        tma_load_2d_pair(sb, mB, fb, bx, by + kb * BK);
        tma_load_2d_pair(sb + 8192, mB, fb, bx + 64, by + kb * BK);
      }
      pipe.advance();
      ++fills;
    }
    return true;
  }

  // ---- unmasked producer (each CTA): all nkb stages of this CTA's halves,
  // each announced by the rank-0 producer as soon as it is issued.
  template <bool A_MN, bool B_MN>
  __device__ __forceinline__ bool produce(const CUtensorMap* mA, const CUtensorMap* mB, int ax,
                                          int ay, int bx, int by, int nkb) {
    for (int kb = 0; kb < nkb; ++kb) {
      if (!wait(smem_u32(&ctl->empty[pipe.stage]), pipe.phase ^ 1u)) return false;
      if (rank == 0) mbar_arrive_expect_tx(smem_u32(&ctl->full[pipe.stage]), 2 * SB);
      const uint32_t fb = in_cta(&ctl->full[pipe.stage], 0);
      const uint32_t sa = smem_u32(smem + pipe.stage * SB);
      const uint32_t sb = sa + PA_BYTES;
      if (!A_MN) {
        tma_load_2d_pair(sa, mA, fb, ax + kb * BK, ay);
      } else {
        tma_load_2d_pair(sa, mA, fb, ax, ay + kb * BK);
        tma_load_2d_pair(sa + 8192, mA, fb, ax + 64, ay + kb * BK);
      }
      if (!B_MN) {
        tma_load_2d_pair(sb, mB, fb, bx + kb * BK, by);
      } else {
        tma_load_2d_pair(sb, mB, fb, bx, by + kb * BK);
        tma_load_2d_pair(sb + 8192, mB, fb, bx + 64, by + kb * BK);
      }
      pipe.advance();
      ++fills;
    }
    return true;
  }

  // ---- unmasked MMA issuer (rank 0): every K step of nkb stages.
  template <bool A_MN, bool B_MN>
  __device__ __forceinline__ bool mma(int nkb) {
    const int acc = tcount & 1;
    if (!wait(smem_u32(&ctl->tempty[acc]), (((uint32_t)tcount >> 1) & 1u) ^ 1u)) return false;
    tc_fence_after();
    const uint32_t d = tmem + acc * BN;
    constexpr uint32_t idesc = idesc_bf16_f32(2 * BM, BN, A_MN, B_MN);
    constexpr uint32_t a_step = A_MN ? 2048 : 32;
    constexpr uint32_t b_step = B_MN ? 2048 : 32;
    const uint64_t ad0 = A_MN ? smem_desc_sw128(smem_u32(smem), 8192, 1024)
                              : smem_desc_sw128(smem_u32(smem), 16, 1024);
    const uint64_t bd0 = B_MN ? smem_desc_sw128(smem_u32(smem) + PA_BYTES, 8192, 1024)
                              : smem_desc_sw128(smem_u32(smem) + PA_BYTES, 16, 1024);
    for (int kb = 0; kb < nkb; ++kb) {
      if (!wait(smem_u32(&ctl->full[pipe.stage]), pipe.phase)) return false;
      tc_fence_after();
      const uint64_t so = (uint64_t)((pipe.stage * SB) >> 4);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        umma_bf16_pair(d, ad0 + so + kk * (a_step >> 4), bd0 + so + kk * (b_step >> 4), idesc,
                       (kb | kk) != 0);
      umma_commit_pair_both(smem_u32(&ctl->empty[pipe.stage]));
      pipe.advance();
      ++fills;
    }
    umma_commit_pair_both(smem_u32(&ctl->tfull[acc]));
    ++tcount;
    return true;
  }

  // ---- MMA issuer (rank 0 only, one thread): consumes the records until
  // REC_LAST; each stage is released to both CTAs' producers by a commit to
  // each CTA's empty barrier, the tile's accumulator to both epilogues.
  template <bool A_MN, bool B_MN>
  __device__ __forceinline__ bool mma_rec() {
    const int acc = tcount & 1;
    if (!wait(smem_u32(&ctl->tempty[acc]), (((uint32_t)tcount >> 1) & 1u) ^ 1u)) return false;
    tc_fence_after();
    const uint32_t d = tmem + acc * BN;
    constexpr uint32_t idesc = idesc_bf16_f32(2 * BM, BN, A_MN, B_MN);
    constexpr uint32_t a_step = A_MN ? 2048 : 32;  // bytes per K=16 step
    constexpr uint32_t b_step = B_MN ? 2048 : 32;
    const uint64_t ad0 = A_MN ? smem_desc_sw128(smem_u32(smem), 8192, 1024)
                              : smem_desc_sw128(smem_u32(smem), 16, 1024);
    const uint64_t bd0 = B_MN ? smem_desc_sw128(smem_u32(smem) + PA_BYTES, 8192, 1024)
                              : smem_desc_sw128(smem_u32(smem) + PA_BYTES, 16, 1024);
    uint32_t issued = 0;
    for (;;) {
      if (!wait(smem_u32(&ctl->full[pipe.stage]), pipe.phase)) return false;
      tc_fence_after();
      const uint32_t rec = *reinterpret_cast<volatile uint32_t*>(&ctl->rec[pipe.stage]);
      const uint64_t so = (uint64_t)((pipe.stage * SB) >> 4);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        if (!(rec & (1u << kk))) continue;
        umma_bf16_pair(d, ad0 + so + kk * (a_step >> 4), bd0 + so + kk * (b_step >> 4), idesc,
                       issued);
        issued = 1;
      }
      umma_commit_pair_both(smem_u32(&ctl->empty[pipe.stage]));
      pipe.advance();
      ++fills;
      if (rec & REC_LAST) break;
    }
    umma_commit_pair_both(smem_u32(&ctl->tfull[acc]));
    ++tcount;
    return true;
  }

  // ---- two products over one staged 128-row B tile (each CTA, lane 0 of
  // warp 0; needs the dual geometry PAIR_DUAL_STAGES x PDUAL_STAGE_BYTES):
  // a stage holds this CTA's 128 rows of each of two A operands (rows ay ..
  // ay+127 of mA0 and mA1) and its 64 of B's 128 rows (rows by .. by+63).
  // The rank-0 MMA thread issues two M = 256, N = 128 products per K step
  // into columns [0, 128) and [128, 256) of one accumulator, so a tile takes
  // 256 TMEM columns and the two accumulators still alternate (the epilogue
  // of a tile overlaps the MMAs of the next), at the shared-memory operand
  // bytes per FLOP of a single-CTA N = 256 product.
  __device__ __forceinline__ bool produce_dual(const CUtensorMap* mA0, const CUtensorMap* mA1,
                                               const CUtensorMap* mB64, int ay, int by, int nkb) {
    static_assert(SB == PDUAL_STAGE_BYTES, "dual products need the dual stage geometry");
    for (int kb = 0; kb < nkb; ++kb) {
      if (!wait(smem_u32(&ctl->empty[pipe.stage]), pipe.phase ^ 1u)) return false;
      if (rank == 0) mbar_arrive_expect_tx(smem_u32(&ctl->full[pipe.stage]), 2 * SB);
      const uint32_t fb = in_cta(&ctl->full[pipe.stage], 0);
      const uint32_t sa = smem_u32(smem + pipe.stage * SB);
      tma_load_2d_pair(sa, mA0, fb, kb * BK, ay);
      tma_load_2d_pair(sa + PA_BYTES, mA1, fb, kb * BK, ay);
      tma_load_2d_pair(sa + 2 * PA_BYTES, mB64, fb, kb * BK, by);
      pipe.advance();
      ++fills;
    }
    return true;
  }
  __device__ __forceinline__ bool mma_dual(int nkb) {
    static_assert(SB == PDUAL_STAGE_BYTES, "dual products need the dual stage geometry");
    const int acc = tcount & 1;
    if (!wait(smem_u32(&ctl->tempty[acc]), (((uint32_t)tcount >> 1) & 1u) ^ 1u)) return false;
    tc_fence_after();
    const uint32_t d0 = tmem + acc * BN;
    const uint32_t d1 = d0 + BN / 2;
    constexpr uint32_t idesc = idesc_bf16_f32(2 * BM, BN / 2, false, false);
    const uint32_t s0 = smem_u32(smem);
    const uint64_t a0 = smem_desc_sw128(s0, 16, 1024);
    const uint64_t a1 = smem_desc_sw128(s0 + PA_BYTES, 16, 1024);
    const uint64_t b0 = smem_desc_sw128(s0 + 2 * PA_BYTES, 16, 1024);
    for (int kb = 0; kb < nkb; ++kb) {
      if (!wait(smem_u32(&ctl->full[pipe.stage]), pipe.phase)) return false;
      tc_fence_after();
      const uint64_t so = (uint64_t)((pipe.stage * SB) >> 4);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t k = so + kk * (32 >> 4);  // 32 bytes per K = 16 step
        umma_bf16_pair(d0, a0 + k, b0 + k, idesc, (kb | kk) != 0);
        umma_bf16_pair(d1, a1 + k, b0 + k, idesc, (kb | kk) != 0);
      }
      umma_commit_pair_both(smem_u32(&ctl->empty[pipe.stage]));
      pipe.advance();
      ++fills;
    }
    umma_commit_pair_both(smem_u32(&ctl->tfull[acc]));
    ++tcount;
    return true;
  }

  // ---- epilogue (both CTAs): this CTA's 128 accumulator rows.
  __device__ __forceinline__ bool epi_acquire(int quarter, uint32_t& taddr) {
    const int acc = tcount & 1;
    if (!wait(smem_u32(&ctl->tfull[acc]), ((uint32_t)tcount >> 1) & 1u)) return false;
    tc_fence_after();
    taddr = tmem + acc * BN + ((uint32_t)(quarter * 32) << 16);
    return true;
  }
  __device__ __forceinline__ void epi_release(int lane) {
    const int acc = tcount & 1;
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(in_cta(&ctl->tempty[acc], 0));
    ++tcount;
  }
};
using PairEngine = PairEngineT<PAIR_STAGES, PSTAGE_BYTES>;

// Bounded wait that ignores the abort flag (used only while draining).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return;
    if ((it & 255u) == 0u && global_timer_ns() - t0 > kWaitLimitNs) return;
  }
}

// Wait limit of a policy's launch: Policy::wait_limit(p) when the policy
// defines it, else kWaitLimitNs.
template <class P, class = void>
struct HasWaitLimit : std::false_type {};
template <class P>
struct HasWaitLimit<P, std::void_t<decltype(P::wait_limit(std::declval<const typename P::Params&>()))>>
    : std::true_type {};
template <class Policy>
__device__ __forceinline__ uint64_t policy_wait_limit(const typename Policy::Params& p) {
  if constexpr (HasWaitLimit<Policy>::value)
    return Policy::wait_limit(p);
  else
    return kWaitLimitNs;
}

// Epilogue warps of a policy: Policy::EPI_WARPS (4 or 8) when it declares
// it, else 4.  With 8, two warps share each TMEM lane quarter; the policy's
// epilogue then takes a fifth argument, 0 or 1, saying which of them it is.
template <class P, class = void>
struct EpiWarps : std::integral_constant<int, 4> {};
template <class P>
struct EpiWarps<P, std::void_t<decltype(P::EPI_WARPS)>>
    : std::integral_constant<int, P::EPI_WARPS> {};
template <class Policy>
constexpr int tc_threads() {
  static_assert(EpiWarps<Policy>::value == 4 || EpiWarps<Policy>::value == 8,
                "4 or 8 epilogue warps");
  return 64 + 32 * EpiWarps<Policy>::value;
}

// The kernel body: set-up, role dispatch, drain, TMEM release.
template <class Policy>
__global__ void __launch_bounds__(tc_threads<Policy>(), 1)
    tc_kernel(const __grid_constant__ typename Policy::Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (base & 1023u)) & 1023u);
  uint8_t* extra = smem + STAGES * STAGE_BYTES;
  Ctl* ctl = reinterpret_cast<Ctl*>(extra + Policy::EXTRA_SMEM);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // launched with programmatic serialization: nothing of global memory is
  // touched before the previous grid in the stream has completed
  grid_dep_launch();
  grid_dep_wait();
  if (!Policy::active(p)) return;  // nothing to do in this launch: skip all set-up

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&ctl->tfull[a]), 1);
      mbar_init(smem_u32(&ctl->tempty[a]), EpiWarps<Policy>::value);
    }
    mbar_init(smem_u32(&ctl->drain), 1);
    ctl->abort = 0;
    ctl->consumed = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) Policy::prefetch(p);
  if (warp == 1) {
    tmem_alloc(smem_u32(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  Engine eng;
  eng.ctl = ctl;
  eng.smem = smem;
  eng.extra = extra;
  eng.tmem = ctl->tmem_base;
  eng.status = p.status;
  eng.wait_ns = policy_wait_limit<Policy>(p);

  if (warp == 0) {
    if (lane == 0) Policy::producer(p, eng);
  } else if (warp == 1) {
    if (lane == 0) {
      Policy::mma(p, eng);
      ctl->consumed = eng.fills;
      // wait until every tcgen05 op this thread issued has completed
      umma_commit(smem_u32(&ctl->drain));
      drain_wait(smem_u32(&ctl->drain), 0);
    }
  } else {
    if constexpr (EpiWarps<Policy>::value == 8)
      Policy::epilogue(p, eng, warp & 3, lane, (warp - 2) >> 2);
    else
      Policy::epilogue(p, eng, warp & 3, lane);
  }
  __syncthreads();
  if (warp == 0 && lane == 0 && ctl->abort) {
    // stage fills issued but never consumed (only after an abort): let the
    // copies land before the CTA exits
    for (int f = ctl->consumed; f < eng.fills; ++f)
      drain_wait(smem_u32(&ctl->full[f % STAGES]), (uint32_t)(f / STAGES) & 1u);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(ctl->tmem_base, TMEM_COLS);
  }
}

// The CTA-pair kernel body: launched with clusters of two CTAs along x.
template <class Policy>
__global__ void __launch_bounds__(THREADS, 1)
    tc_pair_kernel(const __grid_constant__ typename Policy::Params p) {
  using G = PairGeom<Policy>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (base & 1023u)) & 1023u);
  uint8_t* extra = smem + G::NST * G::SB;
  PairCtlT<G::NST>* ctl = reinterpret_cast<PairCtlT<G::NST>*>(extra + Policy::EXTRA_SMEM);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  grid_dep_launch();  // as in tc_kernel
  grid_dep_wait();
  // active() depends only on the parameters and on device values every CTA
  // reads alike, so both CTAs of a pair leave here together or not at all
  if (!Policy::active(p)) return;
  const uint32_t rank = cluster_ctarank();

  if (threadIdx.x == 0) {
    for (int s = 0; s < G::NST; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&ctl->tfull[a]), 1);
      mbar_init(smem_u32(&ctl->tempty[a]), 2 * EPI_THREADS / 32);
    }
    mbar_init(smem_u32(&ctl->drain), 1);
    ctl->abort = 0;
    ctl->consumed = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) Policy::prefetch(p);
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before any remote arrive
  tc_fence_after();

  PairEngineT<G::NST, G::SB> eng;
  eng.ctl = ctl;
  eng.smem = smem;
  eng.extra = extra;
  eng.tmem = ctl->tmem_base;
  eng.status = p.status;
  eng.rank = rank;
  eng.wait_ns = policy_wait_limit<Policy>(p);

  if (warp == 0) {
    if (lane == 0) Policy::producer(p, eng);
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      Policy::mma(p, eng);
      ctl->consumed = eng.fills;
      // every pair MMA this thread issued has completed (they read both
      // CTAs' shared memory, so neither CTA may leave before this)
      umma_commit_pair_own(smem_u32(&ctl->drain));
      drain_wait(smem_u32(&ctl->drain), 0);
    }
  } else {
    Policy::epilogue(p, eng, warp & 3, lane);
  }
  __syncthreads();
  tc_fence_before();
  cluster_sync_all();
  // After an abort, copies issued by either CTA may still be landing (their
  // bytes count on the rank-0 CTA's barriers, which a phase that will never
  // complete cannot report): both CTAs give them a fixed grace period before
  // leaving.  Never taken on the normal path, where every issued stage was
  // consumed by an MMA that waited for all of its bytes.
  const int any_abort =
      ctl->abort | (int)ld_shared_cluster_u32(mapa_shared(smem_u32(&ctl->abort), rank ^ 1u));
  if (any_abort) {
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 2000000ull) {
    }
  }
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(ctl->tmem_base, TMEM_COLS);
  }
}

}  // namespace cce
