// Sparse backward for filtered softmax gradients (CUDA cores).
//
// With the gradient filter on, G = dloss * (p * keep - onehot) keeps only a
// few entries per row ("Cut Your Losses in Large-Vocabulary Language
// Models" research-map entry, §Surprising findings: almost all softmax
// entries vanish; first page §Contribution: those entries carry no
// representable gradient).  When one vocabulary chunk of G holds at most
// `cap` non-zeros (density <= 1/2048), its two contractions are cheaper as
// gathers than as dense tensor-core GEMMs:
//   dE_j  = sum_{i : G_ij != 0} G_ij h_i   (column lists over H_c rows)
//   dH_i += sum_{j : G_ij != 0} G_ij e_j   (row lists over E rows)
// The G producer emits every non-zero (fp32) of a chunk into the chunk's
// list; chunks over capacity take the dense tensor path instead.  The
// decision is taken on the device per chunk, so the host never synchronises.
//
// Both contractions run once, after every chunk's G is known:
//   sparse_count_kernel    entries per column (global walk position) and row
//   (exclusive scans)      column and row offsets (CSR)
//   sparse_scatter_kernel  entries into column order and into row order
//   sparse_de_kernel       each dE row of a sparse chunk: zero, or the
//                          gather over its column list
//   dh_finalize_kernel     each dH row: the dense accumulator plus the
//                          gather over its row list
// A block owns one output row at a time, its threads 8 consecutive elements
// of D each; the row's list is staged in shared memory and its source rows
// are read 8 deep.  Entries of one row or column are summed in an order set
// by atomics, so these sums are not bitwise reproducible run to run.
#pragma once

#include "cce_ptx.cuh"

namespace cce {

struct NzEntry {  // one non-zero of a chunk of G
  int row;        // compact row
  int col;        // column within the chunk
  float g;
  int pad;
};

constexpr int SP_MAX_SEGS = 8;

// Chunk -> (segment, first walk position) for the sparse lists.
struct ChunkMap {
  int n_segs;
  int chunk_begin[SP_MAX_SEGS];  // first global chunk index of each segment
  int width[SP_MAX_SEGS];        // chunk width of each segment
  int live_off[SP_MAX_SEGS];     // first global walk position of each segment
};

__device__ __forceinline__ void chunk_lookup(const ChunkMap& m, int c, int& seg, int& c0) {
  int s = 0;
  while (s + 1 < m.n_segs && c >= m.chunk_begin[s + 1]) ++s;
  seg = s;
  c0 = (c - m.chunk_begin[s]) * m.width[s];
}

// ---- lists -> CSR ------------------------------------------------------------
struct SparseListParams {
  const int* nz_cnt;  // [nch] entries emitted per chunk; > cap: dense chunk, list unused
  int nch, cap;
  const NzEntry* lists;  // [nch][cap]
  ChunkMap cmap;
  int* col_cnt;          // [V_live + 1] entries per global walk position; null: no dE lists
  const int* col_ptr;    // [V_live + 1] exclusive scan of col_cnt
  int2* csorted;         // (compact row, g) in column order
  int* row_cnt;          // [Npad + 1] entries per compact row
  const int* row_ptr;    // [Npad + 1]
  int2* rsorted;         // (segment << 29 | walk position in segment, g) in row order
};

// grid.y = chunk; grid.x strides over the chunk's entries.
__global__ void sparse_count_kernel(const SparseListParams p) {
  const int c = blockIdx.y;
  const int n = p.nz_cnt[c];
  if (n > p.cap) return;
  int seg, c0;
  chunk_lookup(p.cmap, c, seg, c0);
  const int gbase = p.cmap.live_off[seg] + c0;
  const NzEntry* list = p.lists + (size_t)c * p.cap;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x) {
    const NzEntry v = list[e];
    if (p.col_cnt) atomicAdd(&p.col_cnt[gbase + v.col], 1);
    atomicAdd(&p.row_cnt[v.row], 1);
  }
}

// Places every entry at offset + (its count, decremented): the counts end at 0.
__global__ void sparse_scatter_kernel(const SparseListParams p) {
  const int c = blockIdx.y;
  const int n = p.nz_cnt[c];
  if (n > p.cap) return;
  int seg, c0;
  chunk_lookup(p.cmap, c, seg, c0);
  const int gbase = p.cmap.live_off[seg] + c0;
  const NzEntry* list = p.lists + (size_t)c * p.cap;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x) {
    const NzEntry v = list[e];
    const int gv = __float_as_int(v.g);
    if (p.col_cnt) {
      const int gw = gbase + v.col;
      p.csorted[p.col_ptr[gw] + atomicSub(&p.col_cnt[gw], 1) - 1] = make_int2(v.row, gv);
    }
    p.rsorted[p.row_ptr[v.row] + atomicSub(&p.row_cnt[v.row], 1) - 1] =
        make_int2((int)(((unsigned)seg << 29) | (unsigned)(c0 + v.col)), gv);
  }
}

// ---- CSR x dense rows ----------------------------------------------------------
constexpr int GATHER_STAGE = 512;  // list entries staged in shared memory at once
constexpr int GATHER_RANGE = 64;   // output rows whose offsets are loaded together
constexpr int GATHER_MAX_THREADS = 1024;

struct GatherSrc {
  const __nv_bfloat16* src;
  float g;
  int pad;
};

// Adds g * (8 bf16 in h) into acc.
__device__ __forceinline__ void fma8(float (&acc)[8], float g, const uint4 h) {
  acc[0] = fmaf(g, bf16lo(h.x), acc[0]);
  acc[1] = fmaf(g, bf16hi(h.x), acc[1]);
  acc[2] = fmaf(g, bf16lo(h.y), acc[2]);
  acc[3] = fmaf(g, bf16hi(h.y), acc[3]);
  acc[4] = fmaf(g, bf16lo(h.z), acc[4]);
  acc[5] = fmaf(g, bf16hi(h.z), acc[5]);
  acc[6] = fmaf(g, bf16lo(h.w), acc[6]);
  acc[7] = fmaf(g, bf16hi(h.w), acc[7]);
}

// acc += sum over list entries [e0, e1) of g * src[d .. d+8).  Every thread of
// the block calls this with the same e0, e1 (it synchronises the block); a
// thread whose d lies past D passes active = false and only helps staging.
template <class SrcOf>
__device__ __forceinline__ void csr_accumulate(float (&acc)[8], int e0, int e1,
                                               const int2* __restrict__ ent, SrcOf&& src_of,
                                               int d, bool active, GatherSrc* stage) {
  for (int wb = e0; wb < e1; wb += GATHER_STAGE) {
    const int n = min(GATHER_STAGE, e1 - wb);
    __syncthreads();  // the previous window is no longer read
    for (int k = threadIdx.x; k < n; k += blockDim.x) {
      const int2 v = ent[wb + k];
      stage[k] = GatherSrc{src_of(v.x), __int_as_float(v.y), 0};
    }
    __syncthreads();
    if (!active) continue;
    int k = 0;
    for (; k + 8 <= n; k += 8) {
      uint4 h[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) h[u] = __ldg(reinterpret_cast<const uint4*>(stage[k + u].src + d));
#pragma unroll
      for (int u = 0; u < 8; ++u) fma8(acc, stage[k + u].g, h[u]);
    }
    for (; k < n; ++k)
      fma8(acc, stage[k].g, __ldg(reinterpret_cast<const uint4*>(stage[k].src + d)));
  }
}

__device__ __forceinline__ void store_row8(void* row, int d, const float (&a)[8], int fp32_out) {
  if (fp32_out) {
    float4* o = reinterpret_cast<float4*>(static_cast<float*>(row) + d);
    o[0] = make_float4(a[0], a[1], a[2], a[3]);
    o[1] = make_float4(a[4], a[5], a[6], a[7]);
  } else {
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(row) + d) =
        make_uint4(pack_bf16(a[0], a[1]), pack_bf16(a[2], a[3]), pack_bf16(a[4], a[5]),
                   pack_bf16(a[6], a[7]));
  }
}

// dE rows of the chunks taken by the sparse route, indexed by global walk
// position w (segment s, w - live_off[s] within it): zero where the column
// list is empty.  Rows of dense chunks are left to the dense contraction.
struct SparseDEParams {
  const int* col_ptr;  // [V_live + 1]
  const int2* csorted;
  const __nv_bfloat16* Hc;  // [Npad, D]
  long long v_live;
  int D, range;
  const int* nz_cnt;
  int cap;
  ChunkMap cmap;
  const int* vocab_perm;  // concatenated per-segment permutations, or null
  void* dE[SP_MAX_SEGS];
  int fp32_out;
};

__global__ void __launch_bounds__(GATHER_MAX_THREADS) sparse_de_kernel(const SparseDEParams p) {
  __shared__ int sp[GATHER_RANGE + 1];
  __shared__ void* dst[GATHER_RANGE];  // null: written by the dense route
  __shared__ GatherSrc stage[GATHER_STAGE];
  const long long step = (long long)gridDim.x * p.range;
  for (long long r0 = (long long)blockIdx.x * p.range; r0 < p.v_live; r0 += step) {
    const int nr = (int)min((long long)p.range, p.v_live - r0);
    __syncthreads();  // the previous range's offsets are no longer read
    for (int k = threadIdx.x; k <= nr; k += blockDim.x) {
      sp[k] = p.col_ptr[r0 + k];
      if (k < nr) {
        const int w = (int)(r0 + k);
        int s = 0;
        while (s + 1 < p.cmap.n_segs && w >= p.cmap.live_off[s + 1]) ++s;
        const int wl = w - p.cmap.live_off[s];
        void* d = nullptr;
        if (p.nz_cnt[p.cmap.chunk_begin[s] + wl / p.cmap.width[s]] <= p.cap) {
          const size_t row = (size_t)(p.vocab_perm ? p.vocab_perm[w] : wl);
          d = p.fp32_out ? (void*)(static_cast<float*>(p.dE[s]) + row * p.D)
                         : (void*)(static_cast<__nv_bfloat16*>(p.dE[s]) + row * p.D);
        }
        dst[k] = d;
      }
    }
    __syncthreads();
    for (int r = 0; r < nr; ++r) {
      void* out = dst[r];
      if (!out) continue;
      const int e0 = sp[r], e1 = sp[r + 1];
      for (int db = 0; db < p.D; db += blockDim.x * 8) {
        const int d = db + threadIdx.x * 8;
        float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        csr_accumulate(a, e0, e1, p.csorted,
                       [&](int row) { return p.Hc + (size_t)row * p.D; }, d, d < p.D, stage);
        if (d < p.D) store_row8(out, d, a, p.fp32_out);
      }
    }
  }
}

// dH[i] = dH_acc[pos_of_row[i]] + (sparse chunks) sum_j G_ij e_j, in bf16 or
// fp32; 0 for ignored rows, NaN for rows with a bad target.  dH_acc is read
// only when some chunk took the dense route.
struct SparseDHParams {
  const float* dH_acc;    // [Npad, D]
  const int* pos_of_row;  // original row -> compact row; -1 ignored, < -1 bad target
  long long N;
  int D, range;
  void* dH;
  int fp32_out;
  const int* row_ptr;  // [Npad + 1]; null: no row lists
  const int2* rsorted;
  const int* nz_cnt;   // [nch]; null: every chunk took the dense route
  int nch, cap;
  const __nv_bfloat16* E[SP_MAX_SEGS];
  int live_off[SP_MAX_SEGS];
  const int* vocab_perm;  // concatenated per-segment permutations, or null
};

__global__ void __launch_bounds__(GATHER_MAX_THREADS) dh_finalize_kernel(const SparseDHParams p) {
  __shared__ int pj[GATHER_RANGE];
  __shared__ int pe[GATHER_RANGE][2];
  __shared__ GatherSrc stage[GATHER_STAGE];
  __shared__ int dense_any;
  if (threadIdx.x == 0) dense_any = p.nz_cnt ? 0 : 1;
  __syncthreads();
  if (p.nz_cnt)
    for (int c = threadIdx.x; c < p.nch; c += blockDim.x)
      if (p.nz_cnt[c] > p.cap) dense_any = 1;
  __syncthreads();
  const bool use_acc = dense_any != 0;
  auto src_of = [&](int key) {
    const int s = (int)((unsigned)key >> 29), w = key & ((1 << 29) - 1);
    const int loc = p.vocab_perm ? p.vocab_perm[p.live_off[s] + w] : w;
    return p.E[s] + (size_t)loc * p.D;
  };
  const long long step = (long long)gridDim.x * p.range;
  for (long long r0 = (long long)blockIdx.x * p.range; r0 < p.N; r0 += step) {
    const int nr = (int)min((long long)p.range, p.N - r0);
    __syncthreads();
    for (int k = threadIdx.x; k < nr; k += blockDim.x) {
      const int j = p.pos_of_row[r0 + k];
      pj[k] = j;
      pe[k][0] = (j >= 0 && p.row_ptr) ? p.row_ptr[j] : 0;
      pe[k][1] = (j >= 0 && p.row_ptr) ? p.row_ptr[j + 1] : 0;
    }
    __syncthreads();
    for (int r = 0; r < nr; ++r) {
      const int j = pj[r];
      void* out = p.fp32_out ? (void*)(static_cast<float*>(p.dH) + (size_t)(r0 + r) * p.D)
                             : (void*)(static_cast<__nv_bfloat16*>(p.dH) + (size_t)(r0 + r) * p.D);
      for (int db = 0; db < p.D; db += blockDim.x * 8) {
        const int d = db + threadIdx.x * 8;
        const bool act = d < p.D;
        float a[8];
        if (j >= 0 && use_acc && act) {
          const float4* src = reinterpret_cast<const float4*>(p.dH_acc + (size_t)j * p.D + d);
          const float4 u = src[0], v = src[1];
          a[0] = u.x; a[1] = u.y; a[2] = u.z; a[3] = u.w;
          a[4] = v.x; a[5] = v.y; a[6] = v.z; a[7] = v.w;
        } else {
          const float fill = j >= 0 || j == -1 ? 0.f : __int_as_float(0x7fc00000);
#pragma unroll
          for (int k = 0; k < 8; ++k) a[k] = fill;
        }
        if (j >= 0) csr_accumulate(a, pe[r][0], pe[r][1], p.rsorted, src_of, d, act, stage);
        if (act) store_row8(out, d, a, p.fp32_out);
      }
    }
  }
}

// Threads per block for the gathers: 8 elements of D each, whole warps.
inline int gather_threads(long long D) {
  const long long t = ((D / 8 + 31) / 32) * 32;
  return (int)(t < GATHER_MAX_THREADS ? t : GATHER_MAX_THREADS);
}

}  // namespace cce
