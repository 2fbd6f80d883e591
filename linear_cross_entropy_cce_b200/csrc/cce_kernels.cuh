// Kernels of the Cut Cross-Entropy hot path.
//
// Sources (web pages, by title and section):
//   [LM]  "The loss and the mask: Cut Cross-Entropy + FlexAttention (2
//         papers)", part "Cut Your Losses in Large-Vocabulary Language Models
//         (CCE)": §Contribution (indexed dot product for the correct-token
//         logit; blockwise log-sum-exp streamed over vocabulary tiles, logits
//         never written to global memory; backward skips softmax entries
//         below bf16 precision; vocabulary sort), §What transfers to us
//         (valid-row select before the math; two-segment lse by log-add-exp
//         with a -inf dead gap).
//   [MAP] "Cut Your Losses in Large-Vocabulary Language Models" (research
//         map): §Approach (backward recomputes logits blockwise),
//         §Limitations (thread-safe log-add-exp of partial results; Kahan
//         summation for the classifier gradient).
//
// Forward:  compact_kernel -> gather_rows_kernel -> tc_kernel<FwdPolicy>
//           (S = H_c E^T tiles in TMEM, online max/sum-exp per row, one
//           (max, sum) partial per row and vocabulary split) ->
//           fwd_finalize_kernel (log-add-exp of the partials, correct-token
//           logit as an fp32 dot product, loss = lse - z_y).
// Backward: per vocabulary chunk of Vc entries (a bounded slab, never N x V):
//           tc_kernel<GPolicy> recomputes S and writes
//           G = dloss * (softmax * keep - onehot) in bf16 with block masks;
//           tc_kernel<DEPolicy> dE_chunk = G^T H_c (K = rows, on chip);
//           tc_kernel<DHPolicy> dH_acc += G E_chunk (K = chunk);
//           chunks sparse enough skip the last two for the list gathers of
//           cce_sparse.cuh, which run once after all chunks and write dH
//           back to the original rows.
#pragma once

#include <cub/block/block_scan.cuh>

#include "cce_engine.cuh"
#include "cce_sparse.cuh"

namespace cce {

constexpr int MAX_SEGS = 8;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct SegDev {
  long long begin, end;  // logical ids [begin, end)
  int n;                 // live rows (end - begin)
  int tile_off;          // first 256-wide forward tile of this segment
  int live_off;          // offset in the concatenated live vocabulary
  int pad;
  const __nv_bfloat16* E;
};

struct SegTable {
  int n_segs;
  int pad;
  SegDev s[MAX_SEGS];
};

__device__ __forceinline__ int segment_of(const SegTable& t, long long y) {
  for (int s = 0; s < t.n_segs; ++s)
    if (y >= t.s[s].begin && y < t.s[s].end) return s;
  return -1;
}


__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// =====================================================================
// Valid-row select ([LM] §What transfers to us): ordered compaction of the
// rows whose target is not ignore_index.  Single CTA; N int32 reads.
//   pos_of_row[i] = compact index, -1 for ignored rows, -2 for bad targets.
// For the backward it also gathers lse (pre-scaled by log2 e), dloss and
// the target's segment / walk position for each compact row.
// =====================================================================
struct CompactParams {
  const int* y;
  int N;
  int ignore_index;
  SegTable segs;
  int* idx;
  int* pos_of_row;
  int* n_valid;
  int* status;
  // Vocabulary shard: the live vocabulary is this rank's part of a larger
  // one, so a target in [0, V) outside it is a valid row without a one-hot
  // term here (another shard owns it); only targets outside [0, V) are bad.
  int shard;
  long long V;
  // No targets (soft-target KL): y, if given, is only a row mask (rows with
  // y == ignore_index are dropped), and every other row is valid without a
  // one-hot term.
  int no_target;
  // backward extras (nullable)
  const float* lse;
  const float* dloss;
  const int* inv_perm;  // [V_live] walk position of each live row, or null
  float* lse2_c;
  float* dloss_c;
  int* tseg;
  int* tpos;
  const float* lse_t;  // teacher lse (KL), or null
  float* lt2_c;
};

constexpr int COMPACT_THREADS = 1024;

// 0 ignored, 1 valid with its target here, 2 bad target, 3 valid with its
// target in another vocabulary shard.
__device__ __forceinline__ int classify_row(const CompactParams& p, int i, int& seg) {
  if (p.y == nullptr) return 3;
  const int y = p.y[i];
  if (y == p.ignore_index) return 0;
  if (p.no_target) return 3;
  seg = segment_of(p.segs, (long long)y);
  if (seg >= 0) return 1;
  return (p.shard && y >= 0 && (long long)y < p.V) ? 3 : 2;
}

__global__ void __launch_bounds__(COMPACT_THREADS) compact_kernel(const CompactParams p) {
  using Scan = cub::BlockScan<int, COMPACT_THREADS>;
  __shared__ typename Scan::TempStorage tmp;
  const int per = (p.N + COMPACT_THREADS - 1) / COMPACT_THREADS;
  const int lo = threadIdx.x * per;
  const int hi = min(p.N, lo + per);
  int cnt = 0;
  for (int i = lo; i < hi; ++i) {
    int s;
    const int st = classify_row(p, i, s);
    cnt += st == 1 || st == 3;
  }
  int off, total;
  Scan(tmp).ExclusiveSum(cnt, off, total);
  bool bad = false;
  for (int i = lo; i < hi; ++i) {
    int s = -1;
    const int st = classify_row(p, i, s);
    if (st == 1 || st == 3) {
      p.idx[off] = i;
      p.pos_of_row[i] = off;
      if (p.lse2_c) {
        p.lse2_c[off] = p.lse[i] * kLog2e;
        p.dloss_c[off] = p.dloss[i];
        if (p.lt2_c) p.lt2_c[off] = p.lse_t[i] * kLog2e;
        if (st == 1) {
          const int loc = p.y[i] - (int)p.segs.s[s].begin;
          p.tseg[off] = s;
          p.tpos[off] = p.inv_perm ? p.inv_perm[p.segs.s[s].live_off + loc] : loc;
        } else {
          p.tseg[off] = -1;  // no one-hot term in this shard
          p.tpos[off] = -1;
        }
      }
      ++off;
    } else {
      p.pos_of_row[i] = st == 0 ? -1 : -2;
      bad |= st == 2;
    }
  }
  if (bad) atomicOr(p.status, kStatusBadTarget);
  if (threadIdx.x == 0) *p.n_valid = total;
}

// H_c[j] = H[idx[j]] for j < n_valid, zero rows for n_valid <= j < Npad.
// One warp per row, 16-byte vectors.  D is a multiple of 8.
__global__ void gather_rows_kernel(const __nv_bfloat16* __restrict__ H, const int* __restrict__ idx,
                                   const int* __restrict__ n_valid, int Npad, int D,
                                   __nv_bfloat16* __restrict__ Hc) {
  const int lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int nv = *n_valid;
  const int vec = D >> 3;
  for (int j = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; j < Npad; j += nw) {
    uint4* dst = reinterpret_cast<uint4*>(Hc + (size_t)j * D);
    if (j < nv) {
      const uint4* src = reinterpret_cast<const uint4*>(H + (size_t)idx[j] * D);
      for (int v = lane; v < vec; v += 32) dst[v] = __ldg(src + v);
    } else {
      for (int v = lane; v < vec; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
    }
  }
}

// dst[k] = src[perm[k]] for k < rows (vocabulary rows in walk order).
__global__ void gather_perm_rows_kernel(const __nv_bfloat16* __restrict__ src,
                                        const int* __restrict__ perm, int rows, int D,
                                        __nv_bfloat16* __restrict__ dst) {
  const int lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int vec = D >> 3;
  for (int k = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; k < rows; k += nw) {
    const uint4* s = reinterpret_cast<const uint4*>(src + (size_t)perm[k] * D);
    uint4* d = reinterpret_cast<uint4*>(dst + (size_t)k * D);
    for (int v = lane; v < vec; v += 32) d[v] = __ldg(s + v);
  }
}

// =====================================================================
// Forward tile stream ([LM] §Contribution; [MAP] §Approach).
// Work item = (row block mb, vocabulary split): tpi consecutive 256-wide
// vocabulary tiles (tiles never straddle segments).  Items follow the grouped
// order of grouped_item(): split-major within an L2-sized group of row
// blocks, so the CTAs running at the same time share E tiles through L2 and
// re-read row blocks that stay in L2.  Each epilogue thread keeps (m, s) of
// its row in base-2 units:
//   m = max_j z_j log2 e,  s = sum_j 2^(z_j log2 e - m).
// =====================================================================
struct FwdParams {
  CUtensorMap mapA;            // H_c [Npad, D] bf16, box {64, 128}
  CUtensorMap mapB[MAX_SEGS];  // E_s [n_s, D] bf16, box {64, 256} ({64, 128} on CTA pairs)
  SegTable segs;
  int T_v;     // total vocabulary tiles
  int tpi;     // tiles per work item
  int S;       // splits = ceil(T_v / tpi)
  int Npad;    // partial row stride
  int nkb;     // ceil(D / 64)
  const int* n_valid;
  float2* part;  // [S, Npad] (m, s)
  int* colmax;   // ordered-int running max per live vocabulary row, or null
  int* status;
};

// PAIR: on CTA pairs (tc_pair_kernel), 256 x 256 tiles as M = 256 products;
// work unit mbu is a pair of row blocks, 2 mbu (rank 0) and 2 mbu + 1
// (rank 1), and each CTA stages its 128 rows and 128 of the tile's 256 head
// rows and keeps its own 128 accumulator rows.
template <bool PAIR>
struct FwdPolicyT {
  using Params = FwdParams;
  static constexpr int EXTRA_SMEM = 0;
  static __device__ __forceinline__ bool active(const Params&) { return true; }

  template <class F>
  static __device__ __forceinline__ void schedule(const Params& p, F&& f) {
    const int nv = *p.n_valid;
    const int rows_u = PAIR ? 2 * BM : BM;  // rows per work unit
    const int num_u = (nv + rows_u - 1) / rows_u;
    const int num_items = num_u * p.S;
    const int gm = row_group_blocks(num_u, (long long)rows_u * BK * 2 * p.nkb);
    const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    for (int item = unit; item < num_items; item += units) {
      int mbu, split;
      grouped_item(item, num_u, p.S, gm, mbu, split);
      const int t0 = split * p.tpi;
      const int t1 = min(p.T_v, t0 + p.tpi);
      int s = 0;
      for (int t = t0; t < t1; ++t) {
        while (s + 1 < p.segs.n_segs && t >= p.segs.s[s + 1].tile_off) ++s;
        if (!f(mbu, split, t, s, t == t1 - 1, nv)) return;
      }
    }
  }

  static __device__ void prefetch(const Params& p) {
    tma_prefetch_map(&p.mapA);
    for (int s = 0; s < p.segs.n_segs; ++s) tma_prefetch_map(&p.mapB[s]);
  }

  template <class Eng>
  static __device__ void producer(const Params& p, Eng& eng) {
    schedule(p, [&](int mb, int, int t, int s, bool, int) {
      if constexpr (PAIR)
        return eng.template produce<false, false>(
            &p.mapA, &p.mapB[s], 0, (2 * mb + (int)eng.rank) * BM, 0,
            (t - p.segs.s[s].tile_off) * BN + (int)eng.rank * (BN / 2), p.nkb);
      else
        return eng.template produce<false, false>(&p.mapA, &p.mapB[s], 0, mb * BM, 0,
                                                  (t - p.segs.s[s].tile_off) * BN, p.nkb);
    });
  }

  template <class Eng>
  static __device__ void mma(const Params& p, Eng& eng) {
    schedule(p, [&](int, int, int, int, bool, int) {
      return eng.template mma<false, false>(p.nkb);
    });
  }

  template <class Eng>
  static __device__ void epilogue(const Params& p, Eng& eng, int q, int lane) {
    const int row = q * 32 + lane;
    uint32_t rank = 0;
    if constexpr (PAIR) rank = eng.rank;
    float m2 = -INFINITY, sum = 0.f;
    schedule(p, [&](int mbu, int split, int t, int s, bool last, int nv) {
      const int mb = PAIR ? 2 * mbu + (int)rank : mbu;  // this CTA's row block
      uint32_t taddr;
      if (!eng.epi_acquire(q, taddr)) return false;
      const SegDev& sg = p.segs.s[s];
      const int e0 = (t - sg.tile_off) * BN;
      const int valid = min(BN, sg.n - e0);
      const bool row_ok = mb * BM + row < nv;
      for (int c = 0; c < BN / 32; ++c) {
        if (c * 32 >= valid) break;  // uniform over the CTA
        uint32_t r[32];
        tmem_ld32(taddr + c * 32, r);
        float cmax = -INFINITY;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float v = (c * 32 + j < valid) ? __uint_as_float(r[j]) : -INFINITY;
          r[j] = __float_as_uint(v);
          cmax = fmaxf(cmax, v);
        }
        if (p.colmax) {
          int mine = 0;
          const int neg = f32_to_ordered(-INFINITY);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int key = row_ok ? f32_to_ordered(__uint_as_float(r[j])) : neg;
            const int red = __reduce_max_sync(0xffffffffu, key);
            if (lane == j) mine = red;
          }
          if (c * 32 + lane < valid) atomicMax(&p.colmax[sg.live_off + e0 + c * 32 + lane], mine);
        }
        const float mn = fmaxf(m2, cmax * kLog2e);
        float acc = sum * ex2_approx(m2 - mn);
#pragma unroll
        for (int j = 0; j < 32; ++j) acc += ex2_approx(fmaf(__uint_as_float(r[j]), kLog2e, -mn));
        sum = acc;
        m2 = mn;
      }
      eng.epi_release(lane);
      if (last) {
        if (row_ok) p.part[(size_t)split * p.Npad + mb * BM + row] = make_float2(m2, sum);
        m2 = -INFINITY;
        sum = 0.f;
      }
      return true;
    });
  }
};
using FwdPolicy = FwdPolicyT<false>;
using FwdPairPolicy = FwdPolicyT<true>;

// log-add-exp of the split partials, the correct-token logit as an indexed
// dot product in fp32, loss = lse - z_y.  One warp per original row.
struct FinParams {
  const __nv_bfloat16* H;
  const int* y;
  const int* pos_of_row;
  const float2* part;
  SegTable segs;
  int N, D, S, Npad;
  float* loss;  // shard mode: the correct-token logit (0 if another shard owns the target)
  float* lse;   // shard mode: the log-sum-exp over this shard's vocabulary
  int shard;
};

__global__ void fwd_finalize_kernel(const FinParams p) {
  const int lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < p.N; i += nw) {
    const int j = p.pos_of_row[i];
    if (j < 0) {
      if (lane == 0) {
        const float v = j == -1 ? 0.f : __int_as_float(0x7fc00000);
        p.loss[i] = v;
        p.lse[i] = v;
      }
      continue;
    }
    float M = -INFINITY;
    for (int s = lane; s < p.S; s += 32) M = fmaxf(M, p.part[(size_t)s * p.Npad + j].x);
    M = warp_max(M);
    float acc = 0.f;
    for (int s = lane; s < p.S; s += 32) {
      const float2 v = p.part[(size_t)s * p.Npad + j];
      acc += v.y * ex2_approx(v.x - M);
    }
    acc = warp_sum(acc);
    const int y = p.y[i];
    const int sg = segment_of(p.segs, (long long)y);  // < 0 only for another shard's target
    const uint4* h = reinterpret_cast<const uint4*>(p.H + (size_t)i * p.D);
    const uint4* e = reinterpret_cast<const uint4*>(
        sg >= 0 ? p.segs.s[sg].E + (size_t)(y - p.segs.s[sg].begin) * p.D : p.H);
    float dot = 0.f;
    for (int v = lane; sg >= 0 && v < (p.D >> 3); v += 32) {
      const uint4 a = __ldg(h + v), b = __ldg(e + v);
      dot = fmaf(bf16lo(a.x), bf16lo(b.x), dot);
      dot = fmaf(bf16hi(a.x), bf16hi(b.x), dot);
      dot = fmaf(bf16lo(a.y), bf16lo(b.y), dot);
      dot = fmaf(bf16hi(a.y), bf16hi(b.y), dot);
      dot = fmaf(bf16lo(a.z), bf16lo(b.z), dot);
      dot = fmaf(bf16hi(a.z), bf16hi(b.z), dot);
      dot = fmaf(bf16lo(a.w), bf16lo(b.w), dot);
      dot = fmaf(bf16hi(a.w), bf16hi(b.w), dot);
    }
    dot = warp_sum(dot);
    if (lane == 0) {
      const float l = (M + log2f(acc)) * kLn2;
      p.lse[i] = l;
      p.loss[i] = p.shard ? dot : l - dot;
    }
  }
}

// Combine of the vocabulary-parallel forward: per row, the parts of R
// vocabulary shards [R][2][N] (log-sum-exp over the shard, correct-token
// logit or 0) -> lse = log-add-exp over shards ([MAP] §Limitations:
// log-add-exp of partial results; a shard with no ids contributes -inf),
// loss = lse - sum of the logit parts (only the owning shard's is non-zero).
// Ignored rows give 0; a target outside the head's live ranges (outside
// [0, V) or in a dead gap: no shard holds it) gives NaN, as on one GPU.
__global__ void vocab_combine_kernel(const float* __restrict__ parts, int R, const int* __restrict__ y,
                                     int N, int ignore_index, const SegTable t, long long V,
                                     float* __restrict__ loss, float* __restrict__ lse) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < N; i += gridDim.x * blockDim.x) {
    const int yi = y[i];
    if (yi == ignore_index) {
      loss[i] = 0.f;
      lse[i] = 0.f;
      continue;
    }
    if (yi < 0 || (long long)yi >= V || segment_of(t, (long long)yi) < 0) {
      loss[i] = __int_as_float(0x7fc00000);
      lse[i] = __int_as_float(0x7fc00000);
      continue;
    }
    float m = -INFINITY, zy = 0.f;
    for (int r = 0; r < R; ++r) {
      const float* pr = parts + (size_t)r * 2 * N;
      m = fmaxf(m, pr[i]);
      zy += pr[(size_t)N + i];
    }
    float sum = 0.f;
    for (int r = 0; r < R; ++r) sum += expf(parts[(size_t)r * 2 * N + i] - m);
    const float l = m + logf(sum);  // m is finite: the shard holding y_i has ids
    lse[i] = l;
    loss[i] = l - zy;
  }
}

__global__ void colmax_init_kernel(int* colmax, int n) {
  const int neg = f32_to_ordered(-INFINITY);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    colmax[i] = neg;
}
__global__ void colmax_final_kernel(int* colmax, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    reinterpret_cast<float*>(colmax)[i] = ordered_to_f32(colmax[i]);
}

// =====================================================================
// Backward, step 1: recompute S for a vocabulary chunk and write
// G = dloss_i * (p_ij * keep_ij - [j == y_i]) in bf16 ([MAP] §Approach:
// logits recomputed blockwise; [LM] §Contribution: entries below bf16
// precision carry no gradient).  p_ij = 2^(z_ij log2 e - lse_i log2 e).
// keep_ij = p_ij >= eps_keep (element granularity).
// =====================================================================
struct GParams {
  CUtensorMap mapA;  // H_c [Npad, D], box {64, 128}
  CUtensorMap mapB;  // chunk rows of E, K-major, box {64, 256}
  int b_row0;        // map row of the chunk's first vocabulary entry
  int chunk_valid;   // vocabulary entries in this chunk
  int ct;            // 256-wide tiles in the chunk
  int seg, c0;       // segment and walk position of the chunk start
  int Vc;            // G row stride (elements)
  int nkb;
  const int* n_valid;
  const float* lse2_c;
  const float* dloss_c;
  const int* tseg;
  const int* tpos;
  float eps_keep;  // 0: keep everything
  float l2eps;     // log2(eps_keep) (-inf when 0): keep_ij = z_ij log2 e - lse_i log2 e >= l2eps
  __nv_bfloat16* G;
  // Zero-slice masks for the two contractions (zeroed before this launch):
  //   dh_mask[mb * dh_words + g / 32] bit g % 32: some row of row block mb
  //     has a non-zero G entry in chunk columns 16g .. 16g+15;
  //   de_mask[vb * de_words + r / 32] bit r % 32: some entry of compact rows
  //     16r .. 16r+15 is non-zero in chunk columns 128vb .. 128vb+127.
  uint32_t* dh_mask;
  int dh_words;
  uint32_t* de_mask;
  int de_words;
  // Exact tile skip: tile (mb, vt) is not recomputed when
  //   tile_cmax2[vt] - blk_lse2min[mb] < skip_l2,
  // the largest log2 softmax any of its entries can reach (from the
  // forward's column maxima) staying below the keep threshold by a margin;
  // only its one-hot entries are written.  tile_cmax2 null: no skip.
  const float* tile_cmax2;   // per 256-wide tile of this chunk: max colmax * log2 e
  const float* blk_lse2min;  // per 128-row block: min lse * log2 e (rows with dloss != 0)
  float skip_l2;
  // The other mask buffer, cleared by the first launch of this chunk for the
  // next chunk (its last readers, the previous chunk's contractions, are done).
  uint32_t* mask_clear;
  int mask_clear_words;
  // sparse list of this chunk's non-zeros (null: not collected)
  NzEntry* nz_list;
  int* nz_cnt;   // entries emitted (may exceed nz_cap: the chunk is then dense)
  int nz_cap;
  // With a list, the bf16 slab and the masks (the dense fallback) are
  // written only when this chunk is predicted dense: the first chunk, or a
  // chunk after one that overflowed its list.  A mispredicted chunk is
  // recomputed by a second launch with `repair` set, which runs only when
  // the chunk overflowed and its slab was not written.
  const int* prev_nz_cnt;  // previous chunk's count, or null
  int* slab_flag;          // set when this chunk's slab has been written
  int repair;
  // Full classifier gradient (CCE_FULL_DE, GPolicyT<true> only): the
  // unfiltered G of every chunk goes to G_full, which only the dE
  // contraction reads, and de_mask follows G_full; G keeps the filtered
  // values that dH reads.  Written by the first launch of a chunk, not by
  // its repair.
  __nv_bfloat16* G_full;
  // Soft-target KL (GPolicyT<false, true> only): the teacher's rows and
  // classifier, and its lse * log2 e per compact row.  G = dloss (p_s - p_t),
  // an entry kept when either probability reaches the threshold.
  CUtensorMap mapA2;  // H_t,c [Npad, D], box {64, 128}
  CUtensorMap mapB2;  // E_t rows, K-major, box {64, 256}
  // head rows, K-major, as one CTA of a pair stages them: box {64, 128}
  // (cross-entropy, half a 256-id tile) or {64, 64} (KL dual tiles, half a
  // 128-id tile)
  CUtensorMap mapBdual;
  const float* lt2_c;
  // optional per-element keep bits of original rows < debug_rows
  uint32_t* debug_keep;
  int debug_rows;
  int words_per_row;
  const int* idx;
  long long seg_begin;
  const int* perm_seg;  // walk position -> local row, or null
  int* status;
};

// KL (separate heads): each 256-id tile is a teacher and a student N = 256
// product, one per accumulator, so a tile's epilogue waits for both and does
// not overlap the next tile's MMAs.
// PAIR: on CTA pairs (tc_pair_kernel); work unit mbu is a pair of row
// blocks, 2 mbu (rank 0) and 2 mbu + 1 (rank 1), and each CTA keeps its own
// 128 accumulator rows.  Cross-entropy: 256 x 256 tiles, M = 256 products,
// each CTA staging 128 of the tile's 256 head rows.  KL && PAIR (one head
// shared by student and teacher): each 128-id tile is two M = 256, N = 128
// products from one staged head tile (PairEngineT::produce_dual) in one
// accumulator (teacher columns 0..127, student 128..255), so the two
// accumulators alternate and the epilogue overlaps the next tile's MMAs.
template <bool FULL, bool KL = false, bool PAIR = false>
struct GPolicyT {
  static_assert(!(KL && FULL), "the KL producer has no unfiltered classifier gradient");
  using Params = GParams;
  static constexpr bool DUALT = PAIR && KL;  // dual 128-id tiles
  static constexpr int EXTRA_SMEM = 0;
  static constexpr int TN = DUALT ? BN / 2 : BN;  // vocabulary ids per tile
  // stage geometry on CTA pairs
  static constexpr int PAIR_NST = DUALT ? PAIR_DUAL_STAGES : PAIR_STAGES;
  static constexpr int PAIR_SB = DUALT ? PDUAL_STAGE_BYTES : PSTAGE_BYTES;

  // Whether this launch writes the dense fallback (slab + masks), and
  // whether it runs at all (a repair launch usually has nothing to do).
  static __device__ __forceinline__ bool writes_slab(const Params& p) {
    if (!p.nz_list || p.repair) return true;
    return p.prev_nz_cnt == nullptr || *p.prev_nz_cnt > p.nz_cap;
  }
  static __device__ __forceinline__ bool active(const Params& p) {
    return !p.repair || (*p.nz_cnt > p.nz_cap && *p.slab_flag == 0);
  }
  // Exact tile skip of work unit (mbu, vt): every row block of the unit is
  // below the bound (on CTA pairs both blocks, or the one that exists).
  // Producer, MMA issuer and epilogue (of both CTAs) decide alike.
  static __device__ __forceinline__ bool skip(const Params& p, int mbu, int vt, int nv) {
    if (p.tile_cmax2 == nullptr) return false;
    float m;
    if constexpr (PAIR) {
      m = p.blk_lse2min[2 * mbu];
      if (2 * mbu + 1 < (nv + BM - 1) / BM) m = fminf(m, p.blk_lse2min[2 * mbu + 1]);
    } else {
      m = p.blk_lse2min[mbu];
    }
    return p.tile_cmax2[vt] - m < p.skip_l2;
  }

  // f(mbu, vt, nv) for this CTA's (or CTA pair's) work units: mbu a row
  // block, or a pair of row blocks on CTA pairs
  template <class F>
  static __device__ __forceinline__ void schedule(const Params& p, F&& f) {
    const int nv = *p.n_valid;
    const int rows_u = PAIR ? 2 * BM : BM;  // rows per work unit
    const int num_u = (nv + rows_u - 1) / rows_u;
    const int tiles = active(p) ? num_u * p.ct : 0;
    // grouped order (vocabulary-tile-major within L2-sized row groups); the
    // KL producer's A operand is two row blocks (teacher and student)
    const int gm = row_group_blocks(num_u, (long long)rows_u * BK * 2 * p.nkb * (KL ? 2 : 1));
    const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    for (int i = unit; i < tiles; i += units) {
      int mbu, vt;
      grouped_item(i, num_u, p.ct, gm, mbu, vt);
      if (!f(mbu, vt, nv)) return;
    }
  }
  static __device__ void prefetch(const Params& p) {
    tma_prefetch_map(&p.mapA);
    tma_prefetch_map(PAIR ? &p.mapBdual : &p.mapB);
    if constexpr (KL) {
      tma_prefetch_map(&p.mapA2);
      if constexpr (!PAIR) tma_prefetch_map(&p.mapB2);
    }
  }
  template <class Eng>
  static __device__ void producer(const Params& p, Eng& eng) {
    schedule(p, [&](int mb, int vt, int nv) {
      if (skip(p, mb, vt, nv)) return true;
      if constexpr (DUALT) {  // this CTA's 128 rows of each, 64 of the tile's head rows
        return eng.produce_dual(&p.mapA2, &p.mapA, &p.mapBdual, (2 * mb + (int)eng.rank) * BM,
                                p.b_row0 + vt * TN + (int)eng.rank * (TN / 2), p.nkb);
      } else if constexpr (PAIR) {  // this CTA's 128 rows, 128 of the tile's head rows
        return eng.template produce<false, false>(&p.mapA, &p.mapBdual, 0,
                                                  (2 * mb + (int)eng.rank) * BM, 0,
                                                  p.b_row0 + vt * BN + (int)eng.rank * (BN / 2),
                                                  p.nkb);
      } else {
        if constexpr (KL) {  // teacher tile first: it lands in the even accumulator
          if (!eng.template produce<false, false>(&p.mapA2, &p.mapB2, 0, mb * BM, 0,
                                                  p.b_row0 + vt * BN, p.nkb))
            return false;
        }
        return eng.template produce<false, false>(&p.mapA, &p.mapB, 0, mb * BM, 0,
                                                  p.b_row0 + vt * BN, p.nkb);
      }
    });
  }
  template <class Eng>
  static __device__ void mma(const Params& p, Eng& eng) {
    schedule(p, [&](int mb, int vt, int nv) {
      if (skip(p, mb, vt, nv)) return true;
      if constexpr (DUALT) {
        return eng.mma_dual(p.nkb);
      } else {
        if constexpr (KL) {
          if (!eng.template mma<false, false>(p.nkb)) return false;
        }
        return eng.template mma<false, false>(p.nkb);
      }
    });
  }
  template <class Eng>
  static __device__ void epilogue(const Params& p, Eng& eng, int q, int lane) {
    const int row = q * 32 + lane;
    uint32_t rank = 0;
    if constexpr (PAIR) rank = eng.rank;
    const bool slab = writes_slab(p);
    const bool full = FULL && !p.repair;        // this launch writes G_full
    // ... and the dE contraction's masks (none for unfiltered calls)
    const bool de_bits = (FULL ? full : slab) && p.de_mask != nullptr;
    bool emit = p.nz_list != nullptr && !p.repair;  // this warp still lists non-zeros
    if (slab && p.slab_flag && !p.repair && blockIdx.x == 0 && threadIdx.x == 64)
      *p.slab_flag = 1;
    if (!p.repair && p.mask_clear)
      for (int i = blockIdx.x * EPI_THREADS + q * 32 + lane; i < p.mask_clear_words;
           i += gridDim.x * EPI_THREADS)
        p.mask_clear[i] = 0u;
    schedule(p, [&](int mbu, int vt, int nv) {
      const int mb = PAIR ? 2 * mbu + (int)rank : mbu;  // this CTA's row block
      // rank 1's block past the last one (an odd count on CTA pairs): its
      // rows are outside the slab and carry no entries
      const bool blk_live = !PAIR || mb * BM < nv;
      // a skipped tile has no accumulator: no softmax entry is kept in it
      const bool sk = skip(p, mbu, vt, nv);
      uint32_t taddr = 0, tteach = 0;
      if (!sk) {
        if constexpr (DUALT) {
          if (!eng.epi_acquire(q, tteach)) return false;
          taddr = tteach + TN;  // student columns after the teacher's
        } else if constexpr (KL) {
          if (!eng.epi_acquire2(q, tteach, taddr)) return false;
        } else {
          if (!eng.epi_acquire(q, taddr)) return false;
        }
      }
      const int jrow = mb * BM + row;
      const bool ok = jrow < nv;
      const float lse2 = ok ? p.lse2_c[jrow] : 0.f;
      const float lt2 = (KL && ok) ? p.lt2_c[jrow] : 0.f;
      const float dl = ok ? p.dloss_c[jrow] : 0.f;
      const int tcol = (ok && p.tseg[jrow] == p.seg) ? p.tpos[jrow] - p.c0 - vt * TN : -1;
      const int valid = p.chunk_valid - vt * TN;  // valid columns of this tile
      __nv_bfloat16* grow = p.G + (size_t)jrow * p.Vc + vt * TN;
      __nv_bfloat16* frow = FULL ? p.G_full + (size_t)jrow * p.Vc + vt * TN : nullptr;
      const bool dbg = p.debug_keep != nullptr && ok && p.idx[jrow] < p.debug_rows;
      uint32_t half_nz = 0;  // bit h: this row has a non-zero in tile columns 128h..128h+127
      for (int c = 0; c < TN / 32; ++c) {
        uint32_t r[32];
        uint32_t rt[KL ? 32 : 1];  // teacher log2 softmax (KL)
        // keep bits: softmax part retained (p >= eps, decided in base-2 log
        // space; for KL either distribution's), then the non-zero set
        // including the target's one-hot term
        uint32_t kb = 0;
        if (sk) {
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = 0u;
        } else {
          tmem_ld32(taddr + c * 32, r);
          if constexpr (KL) tmem_ld32(tteach + c * 32, rt);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float z2 = fmaf(__uint_as_float(r[j]), kLog2e, -lse2);
            r[j] = __float_as_uint(z2);
            bool keep = z2 >= p.l2eps;
            if constexpr (KL) {
              const float t2 = fmaf(__uint_as_float(rt[j]), kLog2e, -lt2);
              rt[j] = __float_as_uint(t2);
              keep = keep || t2 >= p.l2eps;
            }
            kb |= (keep ? 1u : 0u) << j;
          }
        }
        // softmax part of G at column j (before dloss): p_ij, or p_s - p_t
        auto pval = [&](int j) {
          if constexpr (KL)
            return ex2_approx(__uint_as_float(r[j])) - ex2_approx(__uint_as_float(rt[j]));
          else
            return ex2_approx(__uint_as_float(r[j]));
        };
        const int nvc = min(32, max(0, valid - c * 32));  // valid columns in this 32-chunk
        const uint32_t cm = (ok && dl != 0.f) ? (nvc == 32 ? 0xFFFFFFFFu : ((1u << nvc) - 1u)) : 0u;
        kb &= cm;
        const int tj = tcol - c * 32;
        const uint32_t tb = (tj >= 0 && tj < 32) ? (cm & (1u << tj)) : 0u;
        const uint32_t nzb = kb | tb;  // entries of G that are non-zero
        if ((slab || full) && blk_live) {
          // softmax entries evaluated: the kept ones, or all valid ones for G_full
          const uint32_t ks = full ? cm : kb;
          uint32_t pk[16], pf[FULL ? 16 : 1];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            float gk[2], gf[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const float t = ((tb >> (j + u)) & 1u) ? 1.f : 0.f;
              const float v = ((ks >> (j + u)) & 1u) ? pval(j + u) : 0.f;
              gf[u] = dl * (v - t);
              gk[u] = ((kb >> (j + u)) & 1u) ? gf[u] : (t != 0.f ? -dl : 0.f);
            }
            pk[j >> 1] = pack_bf16(gk[0], gk[1]);
            if constexpr (FULL) pf[j >> 1] = pack_bf16(gf[0], gf[1]);
          }
          if (slab) {
            uint4* dst = reinterpret_cast<uint4*>(grow + c * 32);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            dst[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
            dst[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
            // warp vote: which 16-column slices of this chunk hold any non-zero
            // (unfiltered calls keep no masks: every slice is issued)
            if (p.dh_mask != nullptr) {
              const uint32_t b0 = __ballot_sync(0xffffffffu, (nzb & 0xFFFFu) != 0u);
              const uint32_t b1 = __ballot_sync(0xffffffffu, (nzb >> 16) != 0u);
              if (lane == 0 && (b0 | b1)) {
                const int g = vt * (TN / 16) + c * 2;
                atomicOr(&p.dh_mask[mb * p.dh_words + (g >> 5)],
                         ((b0 ? 1u : 0u) | (b1 ? 2u : 0u)) << (g & 31));
              }
            }
          }
          if constexpr (FULL) {
            if (full) {
              uint4* dst = reinterpret_cast<uint4*>(frow + c * 32);
              dst[0] = make_uint4(pf[0], pf[1], pf[2], pf[3]);
              dst[1] = make_uint4(pf[4], pf[5], pf[6], pf[7]);
              dst[2] = make_uint4(pf[8], pf[9], pf[10], pf[11]);
              dst[3] = make_uint4(pf[12], pf[13], pf[14], pf[15]);
            }
          }
          half_nz |= (de_bits && (full ? (cm | tb) : nzb)) ? (1u << (c >> 2)) : 0u;
        }
        if (emit) {
          // warp-aggregated reservation of this chunk's non-zeros in the list
          const int cnt = __popc(nzb);
          int incl = cnt;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
          }
          const int total = __shfl_sync(0xffffffffu, incl, 31);
          if (total > 0) {
            int base = 0;
            if (lane == 0) base = atomicAdd(p.nz_cnt, total);
            base = __shfl_sync(0xffffffffu, base, 0);
            if (base + total > p.nz_cap) emit = false;  // the chunk goes dense: stop listing
            int pos = base + incl - cnt;
            if (nzb) {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                if (!((nzb >> j) & 1u)) continue;
                const float v = ((kb >> j) & 1u) ? pval(j) : 0.f;
                const float g = dl * (v - (((tb >> j) & 1u) ? 1.f : 0.f));
                if (pos < p.nz_cap) p.nz_list[pos] = NzEntry{jrow, vt * TN + c * 32 + j, g, 0};
                ++pos;
              }
            }
          }
        }
        if (dbg && kb) {
          const int orig = p.idx[jrow];
          for (int j = 0; j < 32; ++j) {
            if (!((kb >> j) & 1u)) continue;
            const int w = p.c0 + vt * TN + c * 32 + j;
            const long long lid = p.seg_begin + (p.perm_seg ? p.perm_seg[w] : w);
            atomicOr(&p.debug_keep[(size_t)orig * p.words_per_row + (lid >> 5)], 1u << (lid & 31));
          }
        }
      }
      if (de_bits) {
        // warp vote per 16-row group for the dE contraction's K slices
#pragma unroll
        for (int h = 0; h < TN / 128; ++h) {
          const uint32_t b = __ballot_sync(0xffffffffu, (half_nz >> h) & 1u);
          if (lane == 0 && b) {
            const int g = mb * (BM / 16) + q * 2;
            atomicOr(&p.de_mask[(vt * (TN / 128) + h) * p.de_words + (g >> 5)],
                     (((b & 0xFFFFu) ? 1u : 0u) | ((b >> 16) ? 2u : 0u)) << (g & 31));
          }
        }
      }
      if (!sk) {
        if constexpr (KL && !PAIR)
          eng.epi_release2(lane);
        else
          eng.epi_release(lane);
      }
      return true;
    });
  }
};

using GPolicy = GPolicyT<false>;
using GPolicyFull = GPolicyT<true>;
using GPolicyKL = GPolicyT<false, true>;
using GPolicyPair = GPolicyT<false, false, true>;
using GPolicyFullPair = GPolicyT<true, false, true>;
using GPolicyKLPair = GPolicyT<false, true, true>;

// =====================================================================
// Backward, step 2: dE_chunk = G^T H_c, K = compact rows, accumulated on
// chip; each output element written once (bf16, fp32, or Kahan-added into
// a bf16 sum with a bf16 compensation: [MAP] §Limitations).
// =====================================================================
struct DEParams {
  CUtensorMap mapA;  // G viewed MN-major: [Npad rows, Vc], box {64, 64}
  CUtensorMap mapB;  // H_c MN-major: [Npad, D], box {64, 64}
  int chunk_valid;
  int mt;  // 128-row vocabulary tiles
  int dt;  // 256-wide D tiles
  int D;
  int c0;
  const int* perm_seg;  // walk position -> local row, or null
  void* dE;             // segment base
  __nv_bfloat16* dE_comp;
  int mode;  // 0 bf16 store, 1 fp32 store, 2 Kahan bf16
  const int* nz_cnt;  // chunk handled by the sparse path when *nz_cnt <= nz_cap
  int nz_cap;
  const uint32_t* mask;  // de_mask of the G producer (K-step mask per vocabulary block)
  int mwords;
  const int* n_valid;
  int* status;
};

// True when no K step of a masked tile is issued (the tile is exactly zero).
// Warp-parallel: one round of loads; every lane of the warp must call it.
__device__ __forceinline__ bool mask_empty(const uint32_t* m, int nkb, int lane) {
  if (!m) return false;
  uint32_t any = 0;
  for (int w = lane; w < ((nkb + 7) >> 3); w += 32) any |= __ldg(m + w);
  return __all_sync(0xffffffffu, any == 0u);
}

// One CTA per 128 x 256 tile of dE (PAIR = false) or one CTA pair per
// 256 x 256 tile (PAIR = true, tcgen05 cta_group::2; the host sets mt to the
// number of vocabulary tiles accordingly).
template <bool PAIR>
struct DEPolicyT {
  using Params = DEParams;
  static constexpr int EXTRA_SMEM = 0;
  static constexpr int ROWS = PAIR ? 2 * BM : BM;  // vocabulary rows per tile
  // a chunk taken by the sparse route has no dense work
  static __device__ __forceinline__ bool active(const Params& p) {
    return !(p.nz_cnt && *p.nz_cnt <= p.nz_cap);
  }
  // K-step masks of the (one or two) 128-row vocabulary blocks of tile vt
  // (null without masks: an unfiltered call issues every K step)
  static __device__ __forceinline__ const uint32_t* mask_lo(const Params& p, int vt) {
    return p.mask ? p.mask + (size_t)(PAIR ? 2 * vt : vt) * p.mwords : nullptr;
  }
  static __device__ __forceinline__ const uint32_t* mask_hi(const Params& p, int vt) {
    return (PAIR && p.mask) ? p.mask + (size_t)(2 * vt + 1) * p.mwords : mask_lo(p, vt);
  }

  template <class F>
  static __device__ __forceinline__ void schedule(const Params& p, F&& f) {
    const int nkb = (*p.n_valid + BK - 1) / BK;
    const int tiles = (p.nz_cnt && *p.nz_cnt <= p.nz_cap) ? 0 : p.mt * p.dt;
    const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    for (int i = unit; i < tiles; i += units) {
      const int vt = i / p.dt;
      if (!f(vt, i - vt * p.dt, nkb)) return;
    }
  }
  static __device__ void prefetch(const Params& p) {
    tma_prefetch_map(&p.mapA);
    tma_prefetch_map(&p.mapB);
  }
  template <class Eng>
  static __device__ void producer(const Params& p, Eng& eng) {
    schedule(p, [&](int vt, int dtile, int nkb) {
      if (p.mask == nullptr) {  // unfiltered: every K step, no records
        if constexpr (PAIR)
          return eng.template produce<true, true>(&p.mapA, &p.mapB, vt * ROWS + (int)eng.rank * BM,
                                                  0, dtile * BN + (int)eng.rank * (BN / 2), 0, nkb);
        else
          return eng.template produce<true, true>(&p.mapA, &p.mapB, vt * BM, 0, dtile * BN, 0, nkb);
      }
      if constexpr (PAIR) {
        return eng.template produce_rec<true, true>(
            &p.mapA, &p.mapB, vt * ROWS + (int)eng.rank * BM, 0, dtile * BN + (int)eng.rank * (BN / 2),
            0, nkb, mask_lo(p, vt), mask_hi(p, vt));
      } else {
        return eng.template produce_rec<true, true>(&p.mapA, &p.mapB, vt * BM, 0, dtile * BN, 0,
                                                    nkb, mask_lo(p, vt));
      }
    });
  }
  template <class Eng>
  static __device__ void mma(const Params& p, Eng& eng) {
    schedule(p, [&](int, int, int nkb) {
      if (nkb == 0) return true;
      if (p.mask == nullptr) return eng.template mma<true, true>(nkb);
      if constexpr (PAIR)
        return eng.template mma_rec<true, true>();
      else
        return eng.template mma_rec<true, true>();
    });
  }
  template <class Eng>
  static __device__ void epilogue(const Params& p, Eng& eng, int q, int lane) {
    const int row = q * 32 + lane;
    uint32_t rank = 0;
    if constexpr (PAIR) rank = eng.rank;
    schedule(p, [&](int vt, int dtile, int nkb) {
      const bool zero = nkb == 0 || (mask_empty(mask_lo(p, vt), nkb, lane) &&
                                     (!PAIR || mask_empty(mask_hi(p, vt), nkb, lane)));
      uint32_t taddr = 0;
      if (nkb > 0 && !eng.epi_acquire(q, taddr)) return false;
      const int r = vt * ROWS + (int)rank * BM + row;
      const bool ok = r < p.chunk_valid;
      const int w = p.c0 + r;
      const size_t local = ok ? (size_t)(p.perm_seg ? p.perm_seg[w] : w) : 0;
      for (int c = 0; c < BN / 32; ++c) {
        const int col0 = dtile * BN + c * 32;
        if (col0 >= p.D) break;
        uint32_t v[32];
        if (!zero) {
          tmem_ld32(taddr + c * 32, v);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0u;
        }
        if (!ok) continue;
        const size_t off = local * p.D + col0;
#pragma unroll
        for (int g8 = 0; g8 < 4; ++g8) {
          if (col0 + g8 * 8 >= p.D) break;
          const float* f = reinterpret_cast<const float*>(v) + g8 * 8;
          if (p.mode == 1) {
            float4* d = reinterpret_cast<float4*>(static_cast<float*>(p.dE) + off + g8 * 8);
            d[0] = make_float4(f[0], f[1], f[2], f[3]);
            d[1] = make_float4(f[4], f[5], f[6], f[7]);
          } else if (p.mode == 0) {
            uint4* d = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dE) + off + g8 * 8);
            *d = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                            pack_bf16(f[6], f[7]));
          } else {
            uint4* ds = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dE) + off + g8 * 8);
            uint4* dc = reinterpret_cast<uint4*>(p.dE_comp + off + g8 * 8);
            const uint4 s4 = *ds, c4 = *dc;
            const uint32_t sw[4] = {s4.x, s4.y, s4.z, s4.w};
            const uint32_t cw[4] = {c4.x, c4.y, c4.z, c4.w};
            uint32_t so[4], co[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              float sv[2] = {bf16lo(sw[k]), bf16hi(sw[k])};
              float cv[2] = {bf16lo(cw[k]), bf16hi(cw[k])};
              float tn[2], cn[2];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const float yv = f[2 * k + u] - cv[u];
                const float t = __bfloat162float(__float2bfloat16_rn(sv[u] + yv));
                cn[u] = (t - sv[u]) - yv;
                tn[u] = t;
              }
              so[k] = pack_bf16(tn[0], tn[1]);
              co[k] = pack_bf16(cn[0], cn[1]);
            }
            *ds = make_uint4(so[0], so[1], so[2], so[3]);
            *dc = make_uint4(co[0], co[1], co[2], co[3]);
          }
        }
      }
      if (nkb > 0) eng.epi_release(lane);
      return true;
    });
  }
};
using DEPolicy = DEPolicyT<false>;
using DEPairPolicy = DEPolicyT<true>;

// =====================================================================
// Backward, step 3: dH_acc[j, :] += G[j, chunk] E_chunk, K = chunk.
// =====================================================================
struct DHParams {
  CUtensorMap mapA;  // G K-major: [Npad, Vc], box {64, 128}
  CUtensorMap mapB;  // chunk rows of E, MN-major: box {64, 64}
  CUtensorMap mapC;  // dH_acc fp32 [Npad, D], box {32, 32}, 128-byte swizzle
  int b_row0;
  int nkb;  // ceil(chunk_valid / 64)
  int dt;
  int D;
  float* dH_acc;  // [Npad, D]
  const int* nz_cnt;  // chunk handled by the sparse path when *nz_cnt <= nz_cap
  int nz_cap;
  const uint32_t* mask;  // dh_mask of the G producer (K-step mask per row block)
  int mwords;
  int mblocks;  // 128-row blocks the mask buffer holds (Npad / 128)
  const int* n_valid;
  int* status;
};

// One CTA per 128 x 256 tile of dH (PAIR = false) or one CTA pair per
// 256 x 256 tile (PAIR = true).  In a pair tile whose second 128-row block
// lies beyond the valid rows, that block's rows (zero or stale G rows) are
// computed and reduced into dH_acc rows that nothing reads (rows >= Npad are
// clipped by the tensor map).
template <bool PAIR>
struct DHPolicyT {
  using Params = DHParams;
  static constexpr int ROWS = PAIR ? 2 * BM : BM;
  static __device__ __forceinline__ bool active(const Params& p) {
    return !(p.nz_cnt && *p.nz_cnt <= p.nz_cap);
  }
  // per epilogue warp: two 32 x 32 fp32 staging tiles for the TMA reduce-add
  static constexpr int EXTRA_SMEM = 4 * 2 * 4096;
  // (null without masks: an unfiltered call issues every K step)
  static __device__ __forceinline__ const uint32_t* mask_lo(const Params& p, int mb) {
    return p.mask ? p.mask + (size_t)(PAIR ? 2 * mb : mb) * p.mwords : nullptr;
  }
  static __device__ __forceinline__ const uint32_t* mask_hi(const Params& p, int mb) {
    // the mask buffer has one entry per 128-row block of Npad
    return (PAIR && p.mask && 2 * mb + 1 < p.mblocks) ? p.mask + (size_t)(2 * mb + 1) * p.mwords
                                                      : mask_lo(p, mb);
  }

  template <class F>
  static __device__ __forceinline__ void schedule(const Params& p, F&& f) {
    const int nv = *p.n_valid;
    const int num_mb = (nv + ROWS - 1) / ROWS;
    const int tiles = (p.nz_cnt && *p.nz_cnt <= p.nz_cap) ? 0 : num_mb * p.dt;
    const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    for (int i = unit; i < tiles; i += units) {
      const int mb = i / p.dt;
      if (!f(mb, i - mb * p.dt, nv)) return;
    }
  }
  static __device__ void prefetch(const Params& p) {
    tma_prefetch_map(&p.mapA);
    tma_prefetch_map(&p.mapB);
    tma_prefetch_map(&p.mapC);
  }
  template <class Eng>
  static __device__ void producer(const Params& p, Eng& eng) {
    schedule(p, [&](int mb, int dtile, int) {
      if (p.mask == nullptr) {  // unfiltered: every K step, no records
        if constexpr (PAIR)
          return eng.template produce<false, true>(&p.mapA, &p.mapB, 0,
                                                   mb * ROWS + (int)eng.rank * BM,
                                                   dtile * BN + (int)eng.rank * BM, p.b_row0, p.nkb);
        else
          return eng.template produce<false, true>(&p.mapA, &p.mapB, 0, mb * BM, dtile * BN,
                                                   p.b_row0, p.nkb);
      }
      if constexpr (PAIR) {
        const int r = (int)eng.rank * BM;
        return eng.template produce_rec<false, true>(&p.mapA, &p.mapB, 0, mb * ROWS + r,
                                                     dtile * BN + r, p.b_row0, p.nkb,
                                                     mask_lo(p, mb), mask_hi(p, mb));
      } else {
        return eng.template produce_rec<false, true>(&p.mapA, &p.mapB, 0, mb * BM, dtile * BN,
                                                     p.b_row0, p.nkb, mask_lo(p, mb));
      }
    });
  }
  template <class Eng>
  static __device__ void mma(const Params& p, Eng& eng) {
    schedule(p, [&](int, int, int) {
      if (p.mask == nullptr) return eng.template mma<false, true>(p.nkb);
      return eng.template mma_rec<false, true>();
    });
  }
  // Each warp adds its 32 accumulator rows into dH_acc 32 columns at a time:
  // tcgen05.ld -> swizzled staging tile in shared memory -> TMA reduce-add
  // (performed in L2), double-buffered so the next chunk is staged while the
  // previous reduction still reads shared memory.  Rows past n_valid hold
  // zeros (their G rows are zero), columns past D are clipped by the map.
  template <class Eng>
  static __device__ void epilogue(const Params& p, Eng& eng, int q, int lane) {
    uint8_t* stage = eng.extra + q * 2 * 4096;
    const uint32_t st0 = smem_u32(stage);
    int nbuf = 0;
    uint32_t rank = 0;
    if constexpr (PAIR) rank = eng.rank;
    schedule(p, [&](int mb, int dtile, int) {
      // nothing to add when no K step of the tile was issued
      const bool zero = mask_empty(mask_lo(p, mb), p.nkb, lane) &&
                        (!PAIR || mask_empty(mask_hi(p, mb), p.nkb, lane));
      uint32_t taddr;
      if (!eng.epi_acquire(q, taddr)) return false;
      const int row0 = mb * ROWS + (int)rank * BM + q * 32;
      // rows at or beyond Npad (the upper half of a pair tile past the end)
      // have no dH_acc rows: nothing to add
      const bool skip = zero || row0 >= p.mblocks * BM;
      for (int c = 0; c < BN / 32 && !skip; ++c) {
        const int col0 = dtile * BN + c * 32;
        if (col0 >= p.D) break;
        uint32_t v[32];
        tmem_ld32(taddr + c * 32, v);
        const int b = nbuf & 1;
        if (lane == 0) bulk_wait_read<1>();  // the reduction that used buffer b is done reading
        __syncwarp();
        uint8_t* row = stage + b * 4096 + lane * 128;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float4 f = make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                                 __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]));
          *reinterpret_cast<float4*>(row + ((k ^ (lane & 7)) << 4)) = f;  // 128-byte swizzle
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_2d(&p.mapC, st0 + b * 4096, col0, row0);
          bulk_commit();
        }
        ++nbuf;
      }
      eng.epi_release(lane);
      return true;
    });
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }
};
using DHPolicy = DHPolicyT<false>;
using DHPairPolicy = DHPolicyT<true>;

// Bounds for the exact tile skip of the G producer.  One warp per output:
//   tile_cmax2[tile_off[s] + t] = log2 e * max colmax over walk positions
//     256t .. 256t+255 of segment s (through the vocabulary permutation);
//   blk_lse2min[b] = min lse * log2 e over the valid compact rows of block b
//     with a non-zero dloss (+inf if none).
struct SkipBoundParams {
  const float* colmax;     // [V_live], segment order
  const int* vocab_perm;   // concatenated per-segment permutations, or null
  int n_segs;
  int live_off[MAX_SEGS], n[MAX_SEGS], tile_off[MAX_SEGS + 1];
  float* tile_cmax2;
  const float* lse2_c;
  const float* dloss_c;
  const int* n_valid;
  int n_blk;
  float* blk_lse2min;
};

__global__ void skip_bounds_kernel(const SkipBoundParams p) {
  const int lane = threadIdx.x & 31;
  const int n_tiles = p.tile_off[p.n_segs];
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < n_tiles + p.n_blk; w += nw) {
    if (w < n_tiles) {
      int s = 0;
      while (s + 1 < p.n_segs && w >= p.tile_off[s + 1]) ++s;
      const int t = w - p.tile_off[s];
      float m = -INFINITY;
      for (int k = lane; k < BN; k += 32) {
        const int wl = t * BN + k;
        if (wl >= p.n[s]) break;
        const int v = p.vocab_perm ? p.vocab_perm[p.live_off[s] + wl] : wl;
        m = fmaxf(m, p.colmax[p.live_off[s] + v]);
      }
      m = warp_max(m);
      if (lane == 0) p.tile_cmax2[w] = m * kLog2e;
    } else {
      const int b = w - n_tiles;
      const int nv = *p.n_valid;
      float m = INFINITY;
      for (int k = lane; k < BM; k += 32) {
        const int j = b * BM + k;
        if (j < nv && p.dloss_c[j] != 0.f) m = fminf(m, p.lse2_c[j]);
      }
      m = -warp_max(-m);
      if (lane == 0) p.blk_lse2min[b] = m;
    }
  }
}

// =====================================================================
// Diagnostic: the tile engine with a stage that never fills.  The producer
// loads nothing, so the MMA issuer's wait for its first stage runs out after
// wait_ns, sets the CTA's abort flag and CCE_STATUS_TIMEOUT; the epilogue,
// waiting for an accumulator, sees the abort and returns; the kernel then
// takes its normal drain and TMEM release path.  No copy or MMA is ever in
// flight.  This is how a wait that cannot complete (a lost copy, a peer that
// never arrives) surfaces: a status bit and a returning launch.
// =====================================================================
struct StallParams {
  int* status;
  unsigned long long wait_ns;
};

struct StallPolicy {
  using Params = StallParams;
  static constexpr int EXTRA_SMEM = 0;
  static __device__ __forceinline__ bool active(const Params&) { return true; }
  static __device__ __forceinline__ uint64_t wait_limit(const Params& p) { return p.wait_ns; }
  static __device__ void prefetch(const Params&) {}
  static __device__ void producer(const Params&, Engine&) {}  // never fills a stage
  static __device__ void mma(const Params&, Engine& eng) { eng.mma<false, false>(1); }
  static __device__ void epilogue(const Params&, Engine& eng, int q, int) {
    uint32_t taddr;
    eng.epi_acquire(q, taddr);
  }
};

// The same on a CTA pair (tc_pair_kernel): the rank-0 MMA issuer's wait for
// a stage runs out, the epilogues of both CTAs wait for an accumulator that
// is never committed until their own limits run out; both CTAs then take the
// abort path of the pair kernel (grace period, cluster barriers, freeing the
// pair's tensor memory).
struct StallPairPolicy {
  using Params = StallParams;
  static constexpr int EXTRA_SMEM = 0;
  static __device__ __forceinline__ bool active(const Params&) { return true; }
  static __device__ __forceinline__ uint64_t wait_limit(const Params& p) { return p.wait_ns; }
  static __device__ void prefetch(const Params&) {}
  template <class Eng>
  static __device__ void producer(const Params&, Eng&) {}  // never fills a stage
  template <class Eng>
  static __device__ void mma(const Params&, Eng& eng) {
    eng.template mma<false, false>(1);
  }
  template <class Eng>
  static __device__ void epilogue(const Params&, Eng& eng, int q, int) {
    uint32_t taddr;
    eng.epi_acquire(q, taddr);
  }
};

// inv[perm[k]] = k for one segment (perm and inv point at the segment's
// slice of the concatenated live vocabulary; entries are segment-local).
__global__ void invert_perm_kernel(const int* __restrict__ perm, int n, int* __restrict__ inv) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < n; k += gridDim.x * blockDim.x)
    inv[perm[k]] = k;
}

}  // namespace cce
