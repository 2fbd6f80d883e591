// Soft-target KL divergence without materialised logits.
//
// "The Defensive Edit: Chunking Cross-Entropy Loss After an OOM Wake-Up
// Call", §The OOM: A 12.2 GB Softmax Wall: a soft KL term between a student
// and a teacher softmax over a 248k vocabulary needs two [positions, V]
// softmaxes, which the page then computes in position chunks.  Here neither
// is ever written: per row
//   KL_i = sum_j p_t,ij (log p_t,ij - log p_s,ij)
//        = A_i - lse_t,i + lse_s,i,   A_i = sum_j p_t,ij (z_t,ij - z_s,ij),
// with z_s = H_s E_s^T, z_t = H_t E_t^T (the same head may serve both).
// The forward streams vocabulary tiles like the cross-entropy forward (the
// log-sum-exp composed blockwise, "Cut Your Losses in Large-Vocabulary
// Language Models", first page §Contribution), each tile as a pair of
// accumulators, teacher then student: per row an online (max, sum) for each
// softmax plus the teacher-weighted sum of z_t - z_s, rescaled with the
// teacher's running max.  The backward (teacher constant) is
// G = dloss (p_s - p_t), produced by GPolicyKL and contracted by the
// cross-entropy path's dE/dH kernels.
#pragma once

#include "cce_kernels.cuh"

namespace cce {

struct KLFwdParams {
  CUtensorMap mapAs, mapAt;  // H_s,c / H_t,c [Npad, D], box {64, 128}
  CUtensorMap mapBs, mapBt;  // E_s / E_t [V, D], box {64, 256}
  int V;
  int T_v;   // 256-id vocabulary tiles
  int tpi;   // tiles per work item
  int S;     // splits
  int Npad;  // partial row stride
  int nkb;
  const int* n_valid;
  float* part;  // [S][5][Npad]: m_t (log2), s_t, w, m_s (log2), s_s
  int* status;
};

// Per-row running state of the KL forward over a split's tiles (base-2
// units): teacher max, sum and teacher-weighted sum of z_t - z_s; student
// max and sum.
struct KLRowState {
  float mt, st, w, ms, ss;
  __device__ __forceinline__ void reset() {
    mt = -INFINITY;
    st = 0.f;
    w = 0.f;
    ms = -INFINITY;
    ss = 0.f;
  }
  // the split's partials of compact row r
  __device__ __forceinline__ void store(const KLFwdParams& p, int split, int r) const {
    float* o = p.part + (size_t)split * 5 * p.Npad + r;
    o[0] = mt;
    o[(size_t)p.Npad] = st;
    o[(size_t)2 * p.Npad] = w;
    o[(size_t)3 * p.Npad] = ms;
    o[(size_t)4 * p.Npad] = ss;
  }
};

// Folds one tile of this thread's row into the running state: teacher logits
// at TMEM address ta, student logits at tb, `valid` (> 0) of TN columns.
template <int TN>
__device__ __forceinline__ void kl_fwd_tile(uint32_t ta, uint32_t tb, int valid, KLRowState& s) {
  for (int c = 0; c < TN / 32; ++c) {
    if (c * 32 >= valid) break;  // uniform over the CTA
    const int nvc = min(32, valid - c * 32);
    uint32_t rt[32], rs[32];
    tmem_ld32(ta + c * 32, rt);
    tmem_ld32(tb + c * 32, rs);
    float cmt = -INFINITY, cms = -INFINITY;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (j < nvc) {
        cmt = fmaxf(cmt, __uint_as_float(rt[j]));
        cms = fmaxf(cms, __uint_as_float(rs[j]));
      }
    }
    const float nt = fmaxf(s.mt, cmt * kLog2e);
    const float sct = ex2_approx(s.mt - nt);
    float at = s.st * sct, aw = s.w * sct;
    const float ns = fmaxf(s.ms, cms * kLog2e);
    float as = s.ss * ex2_approx(s.ms - ns);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (j < nvc) {
        const float zt = __uint_as_float(rt[j]), zs = __uint_as_float(rs[j]);
        const float e = ex2_approx(fmaf(zt, kLog2e, -nt));
        at += e;
        aw = fmaf(e, zt - zs, aw);
        as += ex2_approx(fmaf(zs, kLog2e, -ns));
      }
    }
    s.mt = nt;
    s.st = at;
    s.w = aw;
    s.ms = ns;
    s.ss = as;
  }
}

// Each 256-id tile is a pair of N = 256 products (teacher, then student),
// one per accumulator, so the pair's epilogue waits for both and does not
// overlap the next pair's MMAs.  (Two N = 128 products per 128-id tile from
// one staged head tile, which do overlap, measured slower here on one CTA
// and on CTA pairs alike: this epilogue is light, and N = 128 MMAs do half
// the work per instruction.)
// With CCE_KL_FWD_SPLIT_COLS (default 1) the epilogue has 8 warps, two per
// TMEM lane quarter, each folding 128 of a tile's 256 columns: this epilogue
// does not overlap the MMAs, so halving it shortens every tile.  The two
// column halves keep separate partials (split index 2 s + half), which the
// finalize combines like any other splits.
#ifndef CCE_KL_FWD_SPLIT_COLS
#define CCE_KL_FWD_SPLIT_COLS 1
#endif
constexpr int kKLFwdHalves = CCE_KL_FWD_SPLIT_COLS ? 2 : 1;

struct KLFwdPolicy {
  using Params = KLFwdParams;
  static constexpr int EXTRA_SMEM = 0;
  static constexpr int TN = BN;  // vocabulary ids per tile
  static constexpr int EPI_WARPS = 4 * kKLFwdHalves;
  static __device__ __forceinline__ bool active(const Params&) { return true; }

  template <class F>
  static __device__ __forceinline__ void schedule(const Params& p, F&& f) {
    const int nv = *p.n_valid;
    const int num_mb = (nv + BM - 1) / BM;
    const int num_items = num_mb * p.S;
    // grouped order (see grouped_item); each item re-reads two row blocks
    const int gm = row_group_blocks(num_mb, (long long)BM * BK * 2 * p.nkb * 2);
    for (int item = blockIdx.x; item < num_items; item += gridDim.x) {
      int mb, split;
      grouped_item(item, num_mb, p.S, gm, mb, split);
      const int t0 = split * p.tpi;
      const int t1 = min(p.T_v, t0 + p.tpi);
      for (int t = t0; t < t1; ++t)
        if (!f(mb, split, t, t == t1 - 1, nv)) return;
    }
  }

  static __device__ void prefetch(const Params& p) {
    tma_prefetch_map(&p.mapAs);
    tma_prefetch_map(&p.mapAt);
    tma_prefetch_map(&p.mapBs);
    tma_prefetch_map(&p.mapBt);
  }

  static __device__ void producer(const Params& p, Engine& eng) {
    schedule(p, [&](int mb, int, int t, bool, int) {
      return eng.produce<false, false>(&p.mapAt, &p.mapBt, 0, mb * BM, 0, t * BN, p.nkb) &&
             eng.produce<false, false>(&p.mapAs, &p.mapBs, 0, mb * BM, 0, t * BN, p.nkb);
    });
  }

  static __device__ void mma(const Params& p, Engine& eng) {
    schedule(p, [&](int, int, int, bool, int) {
      return eng.mma<false, false>(p.nkb) && eng.mma<false, false>(p.nkb);
    });
  }

  static __device__ void epilogue(const Params& p, Engine& eng, int q, int lane, int half = 0) {
    constexpr int CW = BN / kKLFwdHalves;  // columns this warp folds
    const int row = q * 32 + lane;
    KLRowState st;
    st.reset();
    schedule(p, [&](int mb, int split, int t, bool last, int nv) {
      uint32_t ta, tb;
      if (!eng.epi_acquire2(q, ta, tb)) return false;
      // (nothing to fold when the tile's valid columns end before this half)
      kl_fwd_tile<CW>(ta + half * CW, tb + half * CW, min(CW, p.V - t * BN - half * CW), st);
      eng.epi_release2(lane);
      if (last) {
        if (mb * BM + row < nv) st.store(p, split * kKLFwdHalves + half, mb * BM + row);
        st.reset();
      }
      return true;
    });
  }
};

// Splits combined per row (one warp per original row): KL = A - lse_t +
// lse_s with A = w / s_t after both are rescaled to the teacher's overall
// max.  Masked rows give 0 in all three outputs.
struct KLFinParams {
  const int* pos_of_row;
  const float* part;
  int N, S, Npad;
  float* kl;
  float* lse_s;
  float* lse_t;
};

__global__ void kl_finalize_kernel(const KLFinParams p) {
  const int lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < p.N; i += nw) {
    const int j = p.pos_of_row[i];
    if (j < 0) {
      if (lane == 0) {
        p.kl[i] = 0.f;
        p.lse_s[i] = 0.f;
        p.lse_t[i] = 0.f;
      }
      continue;
    }
    auto at = [&](int s, int k) { return p.part[((size_t)s * 5 + k) * p.Npad + j]; };
    float Mt = -INFINITY, Ms = -INFINITY;
    for (int s = lane; s < p.S; s += 32) {
      Mt = fmaxf(Mt, at(s, 0));
      Ms = fmaxf(Ms, at(s, 3));
    }
    Mt = warp_max(Mt);
    Ms = warp_max(Ms);
    float St = 0.f, W = 0.f, Ss = 0.f;
    for (int s = lane; s < p.S; s += 32) {
      const float ft = ex2_approx(at(s, 0) - Mt);
      St = fmaf(at(s, 1), ft, St);
      W = fmaf(at(s, 2), ft, W);
      Ss = fmaf(at(s, 4), ex2_approx(at(s, 3) - Ms), Ss);
    }
    St = warp_sum(St);
    W = warp_sum(W);
    Ss = warp_sum(Ss);
    if (lane == 0) {
      const float lt = (Mt + log2f(St)) * kLn2;
      const float ls = (Ms + log2f(Ss)) * kLn2;
      p.lse_t[i] = lt;
      p.lse_s[i] = ls;
      p.kl[i] = W / St - lt + ls;
    }
  }
}

}  // namespace cce
