// Host side of libcce: argument validation, workspace layout, TMA tensor-map
// encoding and kernel launches on the caller's stream.  See include/cce.h for
// the contract of every entry point.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <vector>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cub/device/device_radix_sort.cuh>
#include <cub/device/device_scan.cuh>

#include "../../include/cce.h"
#include "cce_kernels.cuh"
#include "cce_kl.cuh"

using namespace cce;

namespace {

constexpr int kPlanSMs = 148;            // SM count the workspace plan assumes
constexpr size_t kGBudgetBytes = 64ull << 20;   // preferred bf16 G slab (about L2-sized)
constexpr size_t kGCapBytes = 512ull << 20;     // never more than this for the slab
constexpr int64_t kDeWaves = 4;                 // dE tiles per chunk >= this many waves
constexpr size_t kAlign = 256;
// Filtered calls may use vocabulary chunks this many times as wide as
// unfiltered ones (their chunks mostly take the sparse route, which writes no
// slab): fewer launches per step, for a slab and E_c buffers that many times
// larger.  With the programmatic dependent launch the launches cost little,
// so the default is 1 (the same width; 2 saved 0.7% of the Gemma-2-2B-shaped
// step for 201 MiB more scratch).
#ifndef CCE_FILTERED_WIDTH_MULT
#define CCE_FILTERED_WIDTH_MULT 1
#endif
constexpr int64_t kFilteredWidthMult = CCE_FILTERED_WIDTH_MULT;
// Chunk widths are capped so that the bf16 G slab of one chunk (plus the
// sparse lists) stays below an eighth of the bf16 logits, N x V x 2 / 8
// bytes: no buffer of the logits' size class.  Binds only for heads with a
// small V (the Phi-3.5-mini-shaped head: 3584 ids per chunk).
#ifndef CCE_CAP_CHUNK_EIGHTH
#define CCE_CAP_CHUNK_EIGHTH 1
#endif
constexpr bool kCapChunkToEighth = CCE_CAP_CHUNK_EIGHTH != 0;

// The dE / dH contractions of cross-entropy calls run on CTA pairs (256 x 256
// tiles, tcgen05 cta_group::2) unless built with CCE_PAIR_DEDH=0.  Filtered
// soft-target KL calls keep single-CTA tiles: their K steps are skipped when
// a 16-wide slice of G is zero across the tile's rows (or columns), which
// happens less often over 256 of them than over 128 (the KL step's dE went
// from 20 to 34 ms on pairs; the filtered Phi-shaped cross-entropy step, also
// on the dense route, gained 2% on pairs).
#ifndef CCE_PAIR_DEDH
#define CCE_PAIR_DEDH 1
#endif
constexpr bool kPairDEDH = CCE_PAIR_DEDH != 0;
// The cross-entropy G producer runs on CTA pairs (256 x 256 tiles) unless
// built with CCE_PAIR_G=0.
#ifndef CCE_PAIR_G
#define CCE_PAIR_G 1
#endif
// Tensor-core kernels are launched with programmatic stream serialization
// (unless built with CCE_PDL=0): a launch may be scheduled while the
// previous kernel in the stream drains, and its CTAs wait in-kernel
// (griddepcontrol.wait) for that kernel to complete before touching global
// memory, so the gap between dependent launches shrinks; most of the
// backward's launches per chunk exit at once on chunks of the other route.
#ifndef CCE_PDL
#define CCE_PDL 1
#endif
constexpr bool kPDL = CCE_PDL != 0;
constexpr bool kPairG = CCE_PAIR_G != 0;
// The cross-entropy forward runs on CTA pairs (256 x 256 tiles) unless built
// with CCE_PAIR_FWD=0.
#ifndef CCE_PAIR_FWD
#define CCE_PAIR_FWD 1
#endif
constexpr bool kPairFwd = CCE_PAIR_FWD != 0;

size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------- driver API
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 tensor map over a row-major [rows, cols] matrix with the given row
// stride (elements), 128-byte swizzle, zero fill out of bounds.
bool make_map_t(CUtensorMap* m, CUtensorMapDataType dt, uint64_t esize, const void* base,
                uint64_t cols, uint64_t rows, uint64_t ld, uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * esize};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
bool make_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t ld,
              uint32_t box_cols, uint32_t box_rows) {
  return make_map_t(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, cols, rows, ld, box_cols, box_rows);
}

int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  int major = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return -1;
  if (major != 10) return -1;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return sms;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A second stream (per host thread and device) for the permuted-E gathers of
// the backward, so the gather of chunk k+1 overlaps the tensor work of chunk
// k; events order it against the caller's stream (fork at the start, join
// before returning), which also keeps stream capture valid.  Created on first
// use and kept; NULL when creation fails (the gathers then run in order on
// the caller's stream).
struct SideStream {
  cudaStream_t ss;
  cudaEvent_t fork, join, ready[2], freed[2];
};

SideStream* side_stream() {
  constexpr int kMaxDev = 64;
  thread_local SideStream per[kMaxDev];
  thread_local int state[kMaxDev];  // 0 untried, 1 ready, -1 failed
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
  if (state[dev] == 0) {
    SideStream& x = per[dev];
    bool ok = cudaStreamCreateWithFlags(&x.ss, cudaStreamNonBlocking) == cudaSuccess;
    cudaEvent_t* evs[6] = {&x.fork, &x.join, &x.ready[0], &x.ready[1], &x.freed[0], &x.freed[1]};
    for (cudaEvent_t* e : evs) ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
    state[dev] = ok ? 1 : -1;
  }
  return state[dev] == 1 ? &per[dev] : nullptr;
}

// ------------------------------------------------------------ segment table
struct Segs {
  int n = 0;
  cce_segment s[CCE_MAX_SEGMENTS];
  int64_t live = 0;  // V_live
};

int build_segs(const void* E, int64_t V, const cce_segment* segs, int32_t n_segs, Segs& out) {
  if (segs == nullptr || n_segs == 0) {
    if (E == nullptr) return CCE_EINVAL;
    out.n = 1;
    out.s[0] = cce_segment{0, V, E, nullptr, nullptr};
    out.live = V;
    return CCE_OK;
  }
  if (E != nullptr || n_segs < 0 || n_segs > CCE_MAX_SEGMENTS) return CCE_EINVAL;
  int64_t prev_end = 0;
  out.n = n_segs;
  out.live = 0;
  for (int i = 0; i < n_segs; ++i) {
    const cce_segment& g = segs[i];
    if (g.vocab_begin < prev_end || g.vocab_end <= g.vocab_begin || g.vocab_end > V) return CCE_EINVAL;
    if (g.E == nullptr || !aligned16(g.E)) return CCE_EINVAL;
    if (g.vocab_end - g.vocab_begin > (int64_t)INT32_MAX) return CCE_EINVAL;
    prev_end = g.vocab_end;
    out.s[i] = g;
    out.live += g.vocab_end - g.vocab_begin;
  }
  return CCE_OK;
}

SegTable dev_table(const Segs& g, int* T_v) {
  SegTable t;
  memset(&t, 0, sizeof(t));
  t.n_segs = g.n;
  int tiles = 0, live = 0;
  for (int i = 0; i < g.n; ++i) {
    SegDev& d = t.s[i];
    d.begin = g.s[i].vocab_begin;
    d.end = g.s[i].vocab_end;
    d.n = (int)(d.end - d.begin);
    d.tile_off = tiles;
    d.live_off = live;
    d.E = static_cast<const __nv_bfloat16*>(g.s[i].E);
    tiles += (int)cdiv(d.n, BN);
    live += d.n;
  }
  if (T_v) *T_v = tiles;
  return t;
}

bool sizes_ok(int64_t N, int64_t D, int64_t V) {
  return N >= 0 && N <= (int64_t)INT32_MAX - 256 && D > 0 && D % 8 == 0 && D <= 65536 && V > 0 &&
         V <= (int64_t)INT32_MAX - 256;
}

// ------------------------------------------------------------ forward plan
struct FwdPlan {
  int64_t Npad;
  int T_v_max, tpi, S_max;
  size_t off_nvalid, off_idx, off_pos, off_hc, off_part, total;
};

// Vocabulary tiles per forward work item.  Enough items for load balance
// (about 24 per SM), at most 16; and few enough that the E tiles the running
// items stream stay within kFwdInflightBytes of L2: the CTAs (or CTA pairs)
// running at once cover about slots / gm vocabulary splits (gm = work units
// per row group, as the kernel's grouped order forms them), each streaming
// its own tiles.  Longer items let the units that share a split drift
// apart, and a tile the laggards need is then re-read from DRAM (on the
// Llama-shaped head: 18.2 GB per forward at 16 tiles per item, 7.6 GB at 2).
constexpr int64_t kFwdInflightBytes = 32ll << 20;
int fwd_tiles_per_item(int64_t Npad, int64_t D, int64_t T_v, bool pair) {
  const int64_t num_mb = Npad / BM;
  const int64_t units = pair ? cdiv(num_mb, 2) : num_mb;
  const int64_t slots = pair ? kPlanSMs / 2 : kPlanSMs;
  const int64_t unit_bytes = (pair ? 2 * BM : BM) * cdiv(D, BK) * BK * 2;
  const int64_t groups = std::max<int64_t>(1, cdiv(units * unit_bytes, (int64_t)kRowGroupBytes));
  const int64_t gm = std::max<int64_t>(1, cdiv(units, groups));
  const int64_t splits = std::max<int64_t>(1, cdiv(slots, gm));
  const int64_t by_l2 = kFwdInflightBytes / (splits * (int64_t)BN * D * 2);
  const int64_t by_balance = num_mb * T_v / (kPlanSMs * 24);
  return (int)std::max<int64_t>(2, std::min<int64_t>({16, by_l2, by_balance}));
}

FwdPlan plan_fwd(int64_t N, int64_t D, int64_t V, int32_t n_segs) {
  FwdPlan p;
  p.Npad = std::max<int64_t>(BM, cdiv(N, BM) * BM);
  p.T_v_max = (int)(cdiv(V, BN) + std::max(1, (int)n_segs));
  // tiles per item as if the call had the most segments, so the partial
  // buffer (S_max rows of partials) never shrinks as n_segs grows
  p.tpi = fwd_tiles_per_item(p.Npad, D, cdiv(V, BN) + CCE_MAX_SEGMENTS, kPairFwd);
  p.S_max = (int)cdiv(p.T_v_max, p.tpi);
  size_t o = 0;
  p.off_nvalid = o; o += align_up(16);
  p.off_idx = o; o += align_up(sizeof(int) * (size_t)std::max<int64_t>(N, 1));
  p.off_pos = o; o += align_up(sizeof(int) * (size_t)std::max<int64_t>(N, 1));
  p.off_hc = o; o += align_up((size_t)p.Npad * D * 2);
  p.off_part = o; o += align_up((size_t)p.S_max * p.Npad * sizeof(float2));
  p.total = o;
  return p;
}

// ------------------------------------------------------ soft-target KL plan
struct KLFwdPlan {
  int64_t Npad;
  int T_v, tpi, S;
  size_t off_nvalid, off_idx, off_pos, off_hs, off_ht, off_part, total;
};

KLFwdPlan plan_kl_fwd(int64_t N, int64_t D, int64_t V) {
  KLFwdPlan p;
  p.Npad = std::max<int64_t>(BM, cdiv(N, BM) * BM);
  p.T_v = (int)cdiv(V, BN);
  // (the rule of fwd_tiles_per_item measured neutral here, at four times
  // the partial buffer: 4 tiles per item instead of 16 on the 24,576 x
  // 248,320 step)
  const int64_t num_mb = p.Npad / BM;
  p.tpi = (int)std::min<int64_t>(16, std::max<int64_t>(2, num_mb * p.T_v / (kPlanSMs * 24)));
  p.S = (int)cdiv(p.T_v, p.tpi);
  size_t o = 0;
  p.off_nvalid = o; o += align_up(16);
  p.off_idx = o; o += align_up(sizeof(int) * (size_t)std::max<int64_t>(N, 1));
  p.off_pos = o; o += align_up(sizeof(int) * (size_t)std::max<int64_t>(N, 1));
  p.off_hs = o; o += align_up((size_t)p.Npad * D * 2);
  p.off_ht = o; o += align_up((size_t)p.Npad * D * 2);
  // partials per split (and per column half of the epilogue, see KLFwdPolicy)
  p.off_part = o; o += align_up((size_t)p.S * kKLFwdHalves * 5 * p.Npad * sizeof(float));
  p.total = o;
  return p;
}

// ----------------------------------------------------------- backward plan
struct BwdPlan {
  int64_t Npad, Vc;  // Vc: chunk width of unfiltered / Kahan calls
  int64_t Vc_f;      // chunk width of filtered calls (the sparse route is likely)
  size_t off_nvalid, off_idx, off_pos, off_lse2, off_dl, off_tseg, off_tpos, off_inv, off_hc,
      off_dh, off_g, off_ec, off_gfull, off_masks, total;
  int de_words;
  size_t mask_bytes;  // one mask buffer, sized for the wider chunk width
  // sparse backward (filtered gradients)
  int64_t nch_max;
  size_t off_nzcnt, off_lists, off_colc, off_csorted, off_rowc, off_rsorted, off_scan, scan_bytes;
  size_t off_tcmax, off_blkmin;  // tile-skip bounds
  size_t off_htc, off_lt2;       // soft-target KL: teacher rows and lse
  // bytes by the size class of the buffers (see cce_bwd_workspace_parts)
  size_t part_rows, part_vocab, part_logits;
};

// Zero-slice mask words for chunk width vc: dH masks (per 128-row block, one
// bit per 16 columns) and dE masks (per 128-column block, one bit per 16 rows).
size_t mask_bytes_for(int64_t Npad, int64_t vc) {
  return sizeof(uint32_t) * ((size_t)(Npad / BM) * cdiv(vc, 512) + (size_t)(vc / BM) * cdiv(Npad, 512));
}
// Sparse-list capacity of one chunk of width vc: density 1/2048.
int64_t list_cap(int64_t Npad, int64_t vc) { return std::max<int64_t>(4096, Npad * vc / 2048); }

BwdPlan plan_bwd_widths(int64_t N, int64_t D, int64_t V, uint32_t flags, bool kl, int64_t cap_u,
                        int64_t cap_f, int nseg);

// Among chunk widths w in [lo, hi] (multiples of 256), the one that needs the
// fewest rounds of dE tiles over the whole vocabulary: chunks(w) x waves of
// one chunk's tiles (`rows` vocabulary rows per tile, `slots` tiles at once);
// the widest on ties.  Narrowing a chunk below the cap can save a nearly
// empty last wave in every chunk.
int64_t best_dE_width(int64_t V, int64_t D, int64_t lo, int64_t hi, int rows, int slots) {
  int64_t best = hi, best_cost = INT64_MAX;
  for (int64_t w = hi; w >= std::max<int64_t>(BN, lo); w -= BN) {
    const int64_t tiles = cdiv(w, rows) * cdiv(D, BN);
    const int64_t cost = cdiv(V, w) * cdiv(tiles, slots);
    if (cost < best_cost) {
      best_cost = cost;
      best = w;
    }
  }
  return best;
}

// The plan for these sizes.  With kCapChunkToEighth the chunk widths shrink
// (in steps of 256 ids) until the logits-class buffers (the G slab(s) and the
// sparse lists) take less than an eighth of the bf16 logits, N x V x 2 / 8,
// and are then trimmed to the width below that cap whose dE contraction
// wastes the least of its last waves.
// nseg: the head's segments (0: one segment); each adds at most one chunk.
// The chunk widths are chosen as if the call had CCE_MAX_SEGMENTS segments,
// so only the list slots depend on nseg: the workspace size never shrinks as
// nseg grows, and a workspace sized for more segments than a call uses is
// always enough.
BwdPlan plan_bwd(int64_t N, int64_t D, int64_t V, uint32_t flags, bool kl = false, int nseg = 0) {
  constexpr int kWidthSegs = CCE_MAX_SEGMENTS;
  BwdPlan p = plan_bwd_widths(N, D, V, flags, kl, INT64_MAX, INT64_MAX, kWidthSegs);
  const double bound = (double)N * (double)V * 2.0 / 8.0;
  // small problems are left alone: their scratch is a few MB whatever the
  // logits, and narrow chunks would only add launches
  if (!kCapChunkToEighth || bound < (double)(64u << 20) || (double)p.part_logits < bound)
    return plan_bwd_widths(N, D, V, flags, kl, INT64_MAX, INT64_MAX, nseg);
  while ((double)p.part_logits >= bound && p.Vc_f > BN)
    p = plan_bwd_widths(N, D, V, flags, kl, p.Vc_f - BN, p.Vc_f - BN, kWidthSegs);
  // the dE contraction runs on CTA pairs (256-row tiles, kPlanSMs / 2 at
  // once), except the soft-target KL's filtered chunks (single CTAs, 128-row
  // tiles)
  const int64_t wu = best_dE_width(V, D, p.Vc / 2, p.Vc, 2 * BM, kPlanSMs / 2);
  const int64_t wf = kl ? best_dE_width(V, D, p.Vc_f / 2, p.Vc_f, BM, kPlanSMs)
                        : best_dE_width(V, D, p.Vc_f / 2, p.Vc_f, 2 * BM, kPlanSMs / 2);
  return plan_bwd_widths(N, D, V, flags, kl, wu, wf, nseg);
}

// The plan with the unfiltered / filtered chunk widths at most cap_u / cap_f.
BwdPlan plan_bwd_widths(int64_t N, int64_t D, int64_t V, uint32_t flags, bool kl, int64_t cap_u,
                        int64_t cap_f, int nseg) {
  BwdPlan p;
  p.Npad = std::max<int64_t>(BM, cdiv(N, BM) * BM);
  // Vocabulary chunk width: an L2-sized slab, widened so that the dE
  // contraction of one chunk ((Vc / 128) x (D / 256) tiles) fills at least
  // kDeWaves waves of the SMs, within the slab cap.
  const int64_t dt = cdiv(D, BN);
  int64_t vc = (int64_t)(kGBudgetBytes / (2 * (size_t)p.Npad));
  vc = std::max<int64_t>(vc, cdiv(kDeWaves * kPlanSMs * BM, dt));
  vc = std::min<int64_t>(vc, (int64_t)(kGCapBytes / (2 * (size_t)p.Npad)));
  vc = std::min<int64_t>(std::min<int64_t>(16384, cap_u), vc) / BN * BN;
  p.Vc = std::max<int64_t>(BN, std::min<int64_t>(vc, cdiv(V, BN) * BN));
  // Filtered calls: kFilteredWidthMult times as wide, within the slab cap.
  int64_t vf = std::min<int64_t>(kFilteredWidthMult * p.Vc,
                                 (int64_t)(kGCapBytes / (2 * (size_t)p.Npad)));
  vf = std::min<int64_t>(std::min<int64_t>(16384, cap_f), vf) / BN * BN;
  p.Vc_f = std::max<int64_t>(p.Vc, std::min<int64_t>(vf, cdiv(V, BN) * BN));
  const int64_t Vw = p.Vc_f;  // buffers scaled by the chunk width are sized for the wider one
  const size_t n4 = sizeof(int) * (size_t)std::max<int64_t>(N, 1);
  // Carve the workspace; every buffer is counted in the class its size
  // scales with: rows (N, N x D), vocabulary (V, V x D) or the logits (N x V:
  // the bf16 G slabs of one chunk and the sparse lists of all chunks).
  size_t o = 0;
  p.part_rows = p.part_vocab = p.part_logits = 0;
  auto take = [&](size_t bytes, size_t& cls) {
    const size_t at = o;
    o += bytes;
    cls += bytes;
    return at;
  };
  size_t& R = p.part_rows;
  size_t& Vb = p.part_vocab;
  size_t& L = p.part_logits;
  p.off_nvalid = take(align_up(16), R);
  p.off_idx = take(align_up(n4), R);
  p.off_pos = take(align_up(n4), R);
  p.off_lse2 = take(align_up(n4), R);
  p.off_dl = take(align_up(n4), R);
  p.off_tseg = take(align_up(n4), R);
  p.off_tpos = take(align_up(n4), R);
  p.off_inv = take(align_up(sizeof(int) * (size_t)V), Vb);
  p.off_hc = take(align_up((size_t)p.Npad * D * 2), R);
  p.off_dh = take(align_up((size_t)p.Npad * D * 4), R);
  p.off_g = take(align_up((size_t)p.Npad * Vw * 2), L);
  p.off_ec = take(2 * align_up((size_t)Vw * D * 2), Vb);  // two buffers: gather k+1 while k runs
  // CCE_FULL_DE: a second slab with the unfiltered G, read by dE only
  p.off_gfull = take((flags & CCE_FULL_DE) ? align_up((size_t)p.Npad * Vw * 2) : 0, L);
  p.de_words = (int)cdiv(p.Npad, 512);
  p.mask_bytes = mask_bytes_for(p.Npad, Vw);
  // two mask buffers: chunk c uses buffer c % 2 and its G launch clears the other
  p.off_masks = take(2 * align_up(p.mask_bytes), L);
  // sparse path: per chunk a list of up to cap(Vc) non-zeros (density 1/2048);
  // chunk count from the narrower width, list slots for whichever needs more
  // chunks of one call: per segment ceil(n_s / width), at most ceil(V / width)
  // plus one per segment
  const int64_t extra = std::max(1, nseg);
  p.nch_max = cdiv(V, p.Vc) + extra;
  const int64_t slots = std::max(p.nch_max * list_cap(p.Npad, p.Vc),
                                 (cdiv(V, p.Vc_f) + extra) * list_cap(p.Npad, p.Vc_f));
  p.off_nzcnt = take(align_up(sizeof(int) * 2 * (size_t)p.nch_max), Vb);  // counts + slab flags
  p.off_lists = take(align_up(sizeof(NzEntry) * (size_t)slots), L);
  p.off_colc = take(align_up(sizeof(int) * 2 * (size_t)(V + 1)), Vb);  // counts, offsets
  p.off_csorted = take(align_up(sizeof(int2) * (size_t)slots), L);
  p.off_rowc = take(align_up(sizeof(int) * 2 * (size_t)(p.Npad + 1)), R);
  p.off_rsorted = take(align_up(sizeof(int2) * (size_t)slots), L);
  // generous bound on cub's single-pass scan scratch (checked again at run time)
  p.scan_bytes = align_up(sizeof(int) * (size_t)(std::max<int64_t>(V, p.Npad) + 1) / 8 + (1u << 20));
  p.off_scan = take(p.scan_bytes, Vb);
  p.off_tcmax = take(align_up(sizeof(float) * (size_t)(cdiv(V, BN) + CCE_MAX_SEGMENTS)), Vb);
  p.off_blkmin = take(align_up(sizeof(float) * (size_t)(p.Npad / BM)), R);
  p.off_htc = take(kl ? align_up((size_t)p.Npad * D * 2) : 0, R);
  p.off_lt2 = take(kl ? align_up(sizeof(float) * (size_t)std::max<int64_t>(N, 1)) : 0, R);
  p.total = o;
  return p;
}

// ---------------------------------------------------------- diagnostics
enum KernelClass { KC_FWD = 0, KC_G = 1, KC_DE = 2, KC_DH = 3, KC_AUX = 4, KC_SPARSE = 5, KC_N = 6 };

std::atomic<uint64_t> g_launches{0};

struct Timing {
  uint32_t mask = 0;
  std::vector<cudaEvent_t> pool;  // reused across enable cycles
  size_t used = 0;
  std::vector<std::pair<int, size_t>> rec;  // (class, index of the start event)
} g_timing;

cudaEvent_t timing_event() {
  if (g_timing.used == g_timing.pool.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    g_timing.pool.push_back(e);
  }
  return g_timing.pool[g_timing.used++];
}

// Records the start event of a timed launch; returns the record slot or -1.
long timing_begin(int cls, cudaStream_t st) {
  if (!(g_timing.mask & (1u << cls))) return -1;
  const size_t i = g_timing.used;
  cudaEvent_t a = timing_event();
  if (!a || !timing_event()) return -1;
  cudaEventRecord(a, st);
  g_timing.rec.emplace_back(cls, i);
  return (long)i;
}
void timing_end(long slot, cudaStream_t st) {
  if (slot >= 0) cudaEventRecord(g_timing.pool[slot + 1], st);
}

// Raises a kernel's dynamic shared-memory limit once per device (the call
// is not repeated per launch, so launches can be captured into CUDA graphs
// without it).
template <class Policy, bool PAIR, class K>
bool smem_attribute_once(K k, int smem) {
  constexpr int kMaxDev = 64;
  // bit d: set on device d; one word per kernel (policy and launch shape)
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return false;
  const uint64_t bit = 1ull << dev;
  if (done.load(std::memory_order_acquire) & bit) return true;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return false;
  done.fetch_or(bit, std::memory_order_release);
  return true;
}

template <class Policy>
int launch_tc(const typename Policy::Params& prm, int grid, cudaStream_t st, int cls) {
  auto k = tc_kernel<Policy>;
  constexpr int smem = smem_bytes<Policy>();
  static_assert(smem <= 232448, "shared memory per CTA exceeds 227 KB");
  if (!smem_attribute_once<Policy, false>(k, smem)) return CCE_ELAUNCH;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(tc_threads<Policy>(), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = kPDL ? 1 : 0;
  const long slot = timing_begin(cls, st);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k, prm);
  timing_end(slot, st);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? CCE_OK : CCE_ELAUNCH;
}

// Launch of a CTA-pair kernel: clusters of two CTAs along x; `pairs` pairs.
template <class Policy>
int launch_tc_pair(const typename Policy::Params& prm, int pairs, cudaStream_t st, int cls) {
  auto k = tc_pair_kernel<Policy>;
  constexpr int smem = pair_smem_bytes<Policy>();
  static_assert(smem <= 232448, "shared memory per CTA exceeds 227 KB");
  if (!smem_attribute_once<Policy, true>(k, smem)) return CCE_ELAUNCH;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = kPDL ? 2 : 1;
  const long slot = timing_begin(cls, st);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k, prm);
  timing_end(slot, st);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? CCE_OK : CCE_ELAUNCH;
}


// Brackets a plain kernel launch of class `cls` with timing events (when
// that class is being timed); use as  { TimedLaunch t(cls, st); k<<<..>>>(); }
struct TimedLaunch {
  long slot;
  cudaStream_t st;
  TimedLaunch(int cls, cudaStream_t s) : slot(timing_begin(cls, s)), st(s) {}
  ~TimedLaunch() { timing_end(slot, st); }
};

// Called right after every other kernel launch: counts it and checks it.
int launched() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? CCE_OK : CCE_ELAUNCH;
}

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

// Compaction + H_c gather shared by forward and backward.
int run_compaction(const CompactParams& cp, const void* H, int64_t Npad, int64_t D, int sms,
                   __nv_bfloat16* Hc, cudaStream_t st) {
  {
    TimedLaunch tl_(KC_AUX, st);
    compact_kernel<<<1, COMPACT_THREADS, 0, st>>>(cp);
  }
  if (launched() != CCE_OK) return CCE_ELAUNCH;
  {
    TimedLaunch tl_(KC_AUX, st);
    gather_rows_kernel<<<sms * 4, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(H), cp.idx,
                                                cp.n_valid, (int)Npad, (int)D, Hc);
  }
  return launched();
}

}  // namespace

// ------------------------------------------------------------- vocab sort
namespace {
__global__ void target_hist_kernel(const int* y, int N, int ignore_index, SegTable t, float* key) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < N; i += gridDim.x * blockDim.x) {
    const int v = y[i];
    if (v == ignore_index) continue;
    const int s = segment_of(t, (long long)v);
    if (s >= 0) atomicAdd(&key[t.s[s].live_off + (v - (int)t.s[s].begin)], 1.0f);
  }
}
__global__ void iota_kernel(int* a, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) a[i] = i;
}

struct SortPlan {
  size_t off_key, off_key_out, off_ids, off_tmp, tmp_bytes, total;
};
SortPlan plan_sort(int64_t V) {
  SortPlan p;
  size_t o = 0;
  p.off_key = o; o += align_up(sizeof(float) * (size_t)V);
  p.off_key_out = o; o += align_up(sizeof(float) * (size_t)V);
  p.off_ids = o; o += align_up(sizeof(int) * (size_t)V);
  p.off_tmp = o;
  // generous bound on cub's radix-sort scratch (checked again at run time)
  p.tmp_bytes = align_up(3 * sizeof(float) * (size_t)V + (8u << 20));
  o += p.tmp_bytes;
  p.total = o;
  return p;
}
}  // namespace

// =================================================================== C ABI
extern "C" {

int cce_version(void) { return 10000; }

const char* cce_strerror(int code) {
  switch (code) {
    case CCE_OK: return "ok";
    case CCE_EINVAL: return "invalid argument (shape, alignment, segment table or NULL pointer)";
    case CCE_EWORKSPACE: return "workspace missing or too small";
    case CCE_ELAUNCH: return "kernel launch or tensor-map encoding failed";
    case CCE_EDEVICE: return "no sm_100 device or driver entry point unavailable";
    default: return "unknown error";
  }
}

size_t cce_fwd_workspace_size(int64_t N, int64_t D, int64_t V, int32_t n_segs) {
  if (!sizes_ok(N, D, V) || n_segs < 0 || n_segs > CCE_MAX_SEGMENTS) return 0;
  return plan_fwd(N, D, V, n_segs).total;
}

size_t cce_bwd_workspace_size(int64_t N, int64_t D, int64_t V, int32_t n_segs, uint32_t flags) {
  if (!sizes_ok(N, D, V) || n_segs < 0 || n_segs > CCE_MAX_SEGMENTS) return 0;
  return plan_bwd(N, D, V, flags, false, n_segs).total;
}

int cce_bwd_workspace_parts(int64_t N, int64_t D, int64_t V, int32_t n_segs, uint32_t flags,
                            size_t* rows, size_t* vocab, size_t* logits) {
  if (!sizes_ok(N, D, V) || n_segs < 0 || n_segs > CCE_MAX_SEGMENTS || !rows || !vocab || !logits)
    return CCE_EINVAL;
  const BwdPlan p = plan_bwd(N, D, V, flags, false, n_segs);
  *rows = p.part_rows;
  *vocab = p.part_vocab;
  *logits = p.part_logits;
  return CCE_OK;
}

}  // extern "C"

namespace {
// The forward of cce_fwd and of cce_fwd_shard (shard: `loss` receives the
// correct-token logit, 0 for targets another shard owns).
int fwd_impl(const void* H, const void* E, const int32_t* y, int64_t N, int64_t D, int64_t V,
             int32_t ignore_index, const cce_segment* segs, int32_t n_segs, float* loss, float* lse,
             float* colmax, void* workspace, size_t workspace_bytes, int32_t* status, void* stream,
             bool shard) {
  if (!sizes_ok(N, D, V)) return CCE_EINVAL;
  Segs sg;
  if (int rc = build_segs(E, V, segs, n_segs, sg)) return rc;
  if (N == 0) return CCE_OK;
  if (!H || !y || !loss || !lse || !status || !aligned16(H)) return CCE_EINVAL;
  const FwdPlan pl = plan_fwd(N, D, V, n_segs);
  if (!workspace || workspace_bytes < pl.total) return CCE_EWORKSPACE;
  const int sms = device_sms();
  if (sms <= 0 || !encode_fn()) return CCE_EDEVICE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  int T_v = 0;
  const SegTable table = dev_table(sg, &T_v);
  CompactParams cp;
  memset(&cp, 0, sizeof(cp));
  cp.y = y;
  cp.N = (int)N;
  cp.ignore_index = ignore_index;
  cp.segs = table;
  cp.idx = at<int>(workspace, pl.off_idx);
  cp.pos_of_row = at<int>(workspace, pl.off_pos);
  cp.n_valid = at<int>(workspace, pl.off_nvalid);
  cp.status = status;
  cp.shard = shard ? 1 : 0;
  cp.V = V;
  __nv_bfloat16* Hc = at<__nv_bfloat16>(workspace, pl.off_hc);
  if (int rc = run_compaction(cp, H, pl.Npad, D, sms, Hc, st)) return rc;

  if (colmax) {
    colmax_init_kernel<<<sms, 256, 0, st>>>(reinterpret_cast<int*>(colmax), (int)sg.live);
    if (launched()) return CCE_ELAUNCH;
  }

  FwdParams fp;
  memset(&fp, 0, sizeof(fp));
  if (!make_map(&fp.mapA, Hc, D, pl.Npad, D, BK, BM)) return CCE_ELAUNCH;
  // on CTA pairs each CTA stages 128 of a tile's 256 head rows
  for (int s = 0; s < sg.n; ++s)
    if (!make_map(&fp.mapB[s], sg.s[s].E, D, table.s[s].n, D, BK, kPairFwd ? BN / 2 : BN))
      return CCE_ELAUNCH;
  fp.segs = table;
  fp.T_v = T_v;
  fp.tpi = pl.tpi;
  fp.S = (int)cdiv(T_v, pl.tpi);
  fp.Npad = (int)pl.Npad;
  fp.nkb = (int)cdiv(D, BK);
  fp.n_valid = cp.n_valid;
  fp.part = at<float2>(workspace, pl.off_part);
  fp.colmax = reinterpret_cast<int*>(colmax);
  fp.status = status;
  if (kPairFwd) {
    const int64_t items = cdiv(pl.Npad / BM, 2) * fp.S;
    if (int rc = launch_tc_pair<FwdPairPolicy>(fp, (int)std::min<int64_t>(sms / 2, items), st,
                                               KC_FWD))
      return rc;
  } else {
    const int64_t items = (pl.Npad / BM) * fp.S;
    if (int rc = launch_tc<FwdPolicy>(fp, (int)std::min<int64_t>(sms, items), st, KC_FWD))
      return rc;
  }

  FinParams fin;
  fin.H = static_cast<const __nv_bfloat16*>(H);
  fin.y = y;
  fin.pos_of_row = cp.pos_of_row;
  fin.part = fp.part;
  fin.segs = table;
  fin.N = (int)N;
  fin.D = (int)D;
  fin.S = fp.S;
  fin.Npad = fp.Npad;
  fin.loss = loss;
  fin.lse = lse;
  fin.shard = shard ? 1 : 0;
  {
    TimedLaunch tl_(KC_AUX, st);
    fwd_finalize_kernel<<<(int)std::min<int64_t>(cdiv(N, 8), sms * 8), 256, 0, st>>>(fin);
  }
  if (launched()) return CCE_ELAUNCH;
  if (colmax) {
    colmax_final_kernel<<<sms, 256, 0, st>>>(reinterpret_cast<int*>(colmax), (int)sg.live);
    if (launched()) return CCE_ELAUNCH;
  }
  return CCE_OK;
}
}  // namespace

extern "C" {

int cce_fwd(const void* H, const void* E, const int32_t* y, int64_t N, int64_t D, int64_t V,
            int32_t ignore_index, const cce_segment* segs, int32_t n_segs, float* loss, float* lse,
            float* colmax, void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  return fwd_impl(H, E, y, N, D, V, ignore_index, segs, n_segs, loss, lse, colmax, workspace,
                  workspace_bytes, status, stream, false);
}

int cce_fwd_shard(const void* H, const void* E, const int32_t* y, int64_t N, int64_t D, int64_t V,
                  int32_t ignore_index, const cce_segment* segs, int32_t n_segs, float* lse_part,
                  float* zy_part, float* colmax, void* workspace, size_t workspace_bytes,
                  int32_t* status, void* stream) {
  return fwd_impl(H, E, y, N, D, V, ignore_index, segs, n_segs, zy_part, lse_part, colmax,
                  workspace, workspace_bytes, status, stream, true);
}

}  // extern "C"

namespace {
// Soft-target KL extras of the shared backward: the teacher's rows, head and
// lse.  With them, y is only a row mask (0 = dropped row, or NULL) and G is
// dloss (p_s - p_t) on the student (H, E).
struct KLArgs {
  const void* Ht;
  const void* Et;
  const float* lse_t;
};

int bwd_impl(const void* H, const void* E, const int32_t* y, const float* lse, const float* dloss,
            int64_t N, int64_t D, int64_t V, int32_t ignore_index, const cce_segment* segs,
            int32_t n_segs, float filter_eps, const int32_t* vocab_perm, const float* colmax,
            uint32_t flags, void* dH,
            void* dE, void* dE_comp, uint32_t* debug_keep, int64_t debug_rows, void* workspace,
            size_t workspace_bytes, int32_t* status, void* stream, const KLArgs* kl) {
  if (!sizes_ok(N, D, V)) return CCE_EINVAL;
  if (flags & ~(CCE_KAHAN_DE | CCE_FP32_GRADS | CCE_FULL_DE | CCE_VOCAB_SHARD | CCE_FP32_DH))
    return CCE_EINVAL;
  if (kl && (flags & (CCE_FULL_DE | CCE_VOCAB_SHARD))) return CCE_EINVAL;
  const bool full_de = flags & CCE_FULL_DE;
  const bool kahan = flags & CCE_KAHAN_DE;
  const bool fp32 = flags & CCE_FP32_GRADS;        // dE (and dH) in fp32
  const bool fp32_dh = fp32 || (flags & CCE_FP32_DH);  // dH in fp32
  if (kahan && fp32) return CCE_EINVAL;
  Segs sg;
  if (int rc = build_segs(E, V, segs, n_segs, sg)) return rc;
  if (segs == nullptr || n_segs == 0) {
    sg.s[0].dE = dE;
    sg.s[0].dE_comp = dE_comp;
  } else if (dE != nullptr || dE_comp != nullptr) {
    return CCE_EINVAL;
  }
  for (int s = 0; s < sg.n; ++s) {
    if (!sg.s[s].dE || !aligned16(sg.s[s].dE)) return CCE_EINVAL;
    if (kahan && (!sg.s[s].dE_comp || !aligned16(sg.s[s].dE_comp))) return CCE_EINVAL;
  }
  if (debug_keep && (debug_rows < 0 || debug_rows > N)) return CCE_EINVAL;
  if (N == 0) return CCE_OK;
  if (!H || (!y && !kl) || !lse || !dloss || !dH || !status || !aligned16(H) || !aligned16(dH))
    return CCE_EINVAL;
  if (kl && (!kl->Ht || !kl->Et || !kl->lse_t || !aligned16(kl->Ht) || !aligned16(kl->Et)))
    return CCE_EINVAL;
  const BwdPlan pl = plan_bwd(N, D, V, flags, kl != nullptr, segs ? n_segs : 0);
  if (!workspace || workspace_bytes < pl.total) return CCE_EWORKSPACE;
  const int sms = device_sms();
  if (sms <= 0 || !encode_fn()) return CCE_EDEVICE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  int T_v = 0;
  const SegTable table = dev_table(sg, &T_v);
  int* inv = vocab_perm ? at<int>(workspace, pl.off_inv) : nullptr;
  if (vocab_perm) {
    for (int s = 0; s < sg.n; ++s) {
      const int n = table.s[s].n, off = table.s[s].live_off;
      {
        TimedLaunch tl_(KC_AUX, st);
        invert_perm_kernel<<<(int)std::min<int64_t>(cdiv(n, 256), sms * 8), 256, 0, st>>>(
            vocab_perm + off, n, inv + off);
      }
      if (launched()) return CCE_ELAUNCH;
    }
  }
  CompactParams cp;
  memset(&cp, 0, sizeof(cp));
  cp.y = y;
  cp.N = (int)N;
  cp.ignore_index = ignore_index;
  cp.segs = table;
  cp.idx = at<int>(workspace, pl.off_idx);
  cp.pos_of_row = at<int>(workspace, pl.off_pos);
  cp.n_valid = at<int>(workspace, pl.off_nvalid);
  cp.status = status;
  cp.shard = (flags & CCE_VOCAB_SHARD) ? 1 : 0;
  cp.V = V;
  cp.lse = lse;
  cp.dloss = dloss;
  cp.inv_perm = inv;
  cp.lse2_c = at<float>(workspace, pl.off_lse2);
  cp.dloss_c = at<float>(workspace, pl.off_dl);
  cp.tseg = at<int>(workspace, pl.off_tseg);
  cp.tpos = at<int>(workspace, pl.off_tpos);
  if (kl) {
    cp.no_target = 1;
    cp.ignore_index = 0;
    cp.lse_t = kl->lse_t;
    cp.lt2_c = at<float>(workspace, pl.off_lt2);
  }
  __nv_bfloat16* Hc = at<__nv_bfloat16>(workspace, pl.off_hc);
  if (int rc = run_compaction(cp, H, pl.Npad, D, sms, Hc, st)) return rc;
  __nv_bfloat16* Ht_c = kl ? at<__nv_bfloat16>(workspace, pl.off_htc) : nullptr;
  if (kl) {
    {
      TimedLaunch tl_(KC_AUX, st);
      gather_rows_kernel<<<sms * 4, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(kl->Ht), cp.idx,
                                                  cp.n_valid, (int)pl.Npad, (int)D, Ht_c);
    }
    if (launched()) return CCE_ELAUNCH;
  }
  float* dH_acc = at<float>(workspace, pl.off_dh);
  if (cudaMemsetAsync(dH_acc, 0, (size_t)pl.Npad * D * 4, st) != cudaSuccess) return CCE_ELAUNCH;
  const int words = (int)cdiv(V, 32);
  if (debug_keep && debug_rows > 0 &&
      cudaMemsetAsync(debug_keep, 0, (size_t)debug_rows * words * 4, st) != cudaSuccess)
    return CCE_ELAUNCH;

  __nv_bfloat16* G = at<__nv_bfloat16>(workspace, pl.off_g);
  __nv_bfloat16* G_full = full_de ? at<__nv_bfloat16>(workspace, pl.off_gfull) : nullptr;
  uint32_t* masks = at<uint32_t>(workspace, pl.off_masks);
  const size_t mask_stride = align_up(pl.mask_bytes) / sizeof(uint32_t);
  if (cudaMemsetAsync(masks, 0, 2 * align_up(pl.mask_bytes), st) != cudaSuccess) return CCE_ELAUNCH;
  __nv_bfloat16* Ec = at<__nv_bfloat16>(workspace, pl.off_ec);
  // chunk width of this call: wider when filtering can take the sparse route
  const bool wide = filter_eps > 0.f && !kahan;
  // (the soft-target KL's filtered chunks keep single-CTA tiles: see kPairDEDH)
  const bool pair_dedh = kPairDEDH && (filter_eps <= 0.f || kl == nullptr);
  // zero-slice masks only pay where G has zeros: filtered calls
  const bool use_masks = filter_eps > 0.f;
  const int Vc = (int)(wide ? pl.Vc_f : pl.Vc);
  const int dh_words = (int)cdiv(Vc, 512);
  const int dt = (int)cdiv(D, BN);
  const int nkbD = (int)cdiv(D, BK);
  const int mbs = (int)(pl.Npad / BM);
  const float eps_keep = filter_eps > 0.f ? filter_eps * (1.0f - 1.0f / 256.0f) : 0.f;
  // Sparse contractions for filtered gradients (chunks with at most `cap`
  // non-zeros; the Kahan path stays on the deterministic dense route).
  // dH may take the sparse route whenever filtering is on; dE only when it is
  // filtered too (not CCE_FULL_DE).
  // exact tile skip from the forward's column maxima (not for FullC, whose
  // dE needs every entry)
  const bool tile_skip = colmax != nullptr && filter_eps > 0.f && !full_de && !kl;
  float* tile_cmax2 = at<float>(workspace, pl.off_tcmax);
  float* blk_lse2min = at<float>(workspace, pl.off_blkmin);
  int tile_off[CCE_MAX_SEGMENTS + 1];
  tile_off[0] = 0;
  for (int s = 0; s < sg.n; ++s) tile_off[s + 1] = tile_off[s] + (int)cdiv(table.s[s].n, BN);
  if (tile_skip) {
    SkipBoundParams bp;
    memset(&bp, 0, sizeof(bp));
    bp.colmax = colmax;
    bp.vocab_perm = vocab_perm;
    bp.n_segs = sg.n;
    for (int s = 0; s < sg.n; ++s) {
      bp.live_off[s] = table.s[s].live_off;
      bp.n[s] = table.s[s].n;
    }
    for (int s = 0; s <= sg.n; ++s) bp.tile_off[s] = tile_off[s];
    bp.tile_cmax2 = tile_cmax2;
    bp.lse2_c = cp.lse2_c;
    bp.dloss_c = cp.dloss_c;
    bp.n_valid = cp.n_valid;
    bp.n_blk = (int)(pl.Npad / BM);
    bp.blk_lse2min = blk_lse2min;
    const int64_t warps = tile_off[sg.n] + bp.n_blk;
    {
      TimedLaunch tl_(KC_AUX, st);
      skip_bounds_kernel<<<(int)std::min<int64_t>(cdiv(warps, 8), sms * 8), 256, 0, st>>>(bp);
    }
    if (launched()) return CCE_ELAUNCH;
  }
  bool sparse = filter_eps > 0.f && !kahan;
  for (int s = 0; s < sg.n; ++s) sparse = sparse && table.s[s].n < (1 << 29);
  const bool sparse_de = sparse && !full_de;
  const int cap = (int)list_cap(pl.Npad, Vc);
  int* nz_cnt = at<int>(workspace, pl.off_nzcnt);
  NzEntry* lists = at<NzEntry>(workspace, pl.off_lists);
  const int64_t v_live = sg.live;
  int* col_cnt = at<int>(workspace, pl.off_colc);
  int* col_ptr = col_cnt + (v_live + 1);
  int2* csorted = at<int2>(workspace, pl.off_csorted);
  int* row_cnt = at<int>(workspace, pl.off_rowc);
  int* row_ptr = row_cnt + (pl.Npad + 1);
  int2* rsorted = at<int2>(workspace, pl.off_rsorted);
  int* slab_flag = nz_cnt + pl.nch_max;
  if (sparse && cudaMemsetAsync(nz_cnt, 0, sizeof(int) * 2 * pl.nch_max, st) != cudaSuccess)
    return CCE_ELAUNCH;
  ChunkMap cmap;
  memset(&cmap, 0, sizeof(cmap));
  cmap.n_segs = sg.n;
  for (int s = 0; s < sg.n; ++s) cmap.live_off[s] = table.s[s].live_off;

  GParams gp;
  DEParams ep;
  DHParams hp;
  memset(&gp, 0, sizeof(gp));
  memset(&ep, 0, sizeof(ep));
  memset(&hp, 0, sizeof(hp));
  if (!make_map(&gp.mapA, Hc, D, pl.Npad, D, BK, BM)) return CCE_ELAUNCH;
  // soft-target KL with one head for student and teacher: dual 128-id
  // tiles on CTA pairs (GPolicyKLPair)
  const bool kl_pair = kl != nullptr && kl->Et == E;
  const bool pair_g = kPairG && kl == nullptr;  // cross-entropy G on CTA pairs
  if (kl) {
    if (!make_map(&gp.mapA2, Ht_c, D, pl.Npad, D, BK, BM)) return CCE_ELAUNCH;
    if (!make_map(&gp.mapB2, kl->Et, D, V, D, BK, BN)) return CCE_ELAUNCH;
    gp.lt2_c = cp.lt2_c;
  }
  if (!make_map(&ep.mapA, full_de ? G_full : G, Vc, pl.Npad, Vc, 64, 64)) return CCE_ELAUNCH;
  if (!make_map(&ep.mapB, Hc, D, pl.Npad, D, 64, 64)) return CCE_ELAUNCH;
  if (!make_map(&hp.mapA, G, Vc, pl.Npad, Vc, BK, BM)) return CCE_ELAUNCH;
  if (!make_map_t(&hp.mapC, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dH_acc, D, pl.Npad, D, 32, 32))
    return CCE_ELAUNCH;

  // the chunk list: per segment, equal chunks (multiples of 256) so the last
  // one is not a sliver
  struct ChunkRef {
    int s, c0, cv;
  };
  std::vector<ChunkRef> chunks;
  for (int s = 0; s < sg.n; ++s) {
    const int ns = table.s[s].n;
    const int nch = (int)cdiv(ns, Vc);
    const int cw = (int)std::min<int64_t>(Vc, cdiv(cdiv(ns, nch), BN) * BN);
    cmap.chunk_begin[s] = (int)chunks.size();
    cmap.width[s] = cw;
    for (int c0 = 0; c0 < ns; c0 += cw) chunks.push_back({s, c0, std::min(cw, ns - c0)});
  }
  const int n_chunks = (int)chunks.size();
  __nv_bfloat16* Ecb[2] = {Ec, Ec + align_up((size_t)Vc * D * 2) / sizeof(__nv_bfloat16)};
  // permuted walk: chunk k's E rows gathered into Ecb[k % 2] (on the side
  // stream one chunk ahead when there is one)
  SideStream* side = vocab_perm ? side_stream() : nullptr;
  auto gather = [&](int k, cudaStream_t gs) -> int {
    const ChunkRef& c = chunks[k];
    {
      TimedLaunch tl_(KC_AUX, gs);
      gather_perm_rows_kernel<<<sms * 4, 256, 0, gs>>>(
          static_cast<const __nv_bfloat16*>(sg.s[c.s].E), vocab_perm + table.s[c.s].live_off + c.c0,
          c.cv, (int)D, Ecb[side ? (k & 1) : 0]);
    }
    return launched();
  };
  if (side) {
    if (cudaEventRecord(side->fork, st) != cudaSuccess ||
        cudaStreamWaitEvent(side->ss, side->fork, 0) != cudaSuccess)
      return CCE_ELAUNCH;
  }
  auto do_chunk = [&](const int chunk) -> int {
    const int s = chunks[chunk].s, c0 = chunks[chunk].c0, cv = chunks[chunk].cv;
    const int ns = table.s[s].n;
    const int* perm_seg = vocab_perm ? vocab_perm + table.s[s].live_off : nullptr;
    // segKhalf: the head rows one CTA of a pair stages, 128 of a cross-entropy
    // tile's 256 or 64 of a KL dual tile's 128
    CUtensorMap segK, segMN, segKhalf;
    int row0 = c0;
    if (perm_seg) {
      if (side) {
        if (chunk == 0) {
          if (int rc = gather(0, side->ss)) return rc;
          if (cudaEventRecord(side->ready[0], side->ss) != cudaSuccess) return CCE_ELAUNCH;
        }
        if (chunk + 1 < n_chunks) {
          // buffer (chunk+1) % 2 was last read by the dH contraction of chunk - 1
          if (chunk >= 1 && cudaStreamWaitEvent(side->ss, side->freed[(chunk + 1) & 1], 0) != cudaSuccess)
            return CCE_ELAUNCH;
          if (int rc = gather(chunk + 1, side->ss)) return rc;
          if (cudaEventRecord(side->ready[(chunk + 1) & 1], side->ss) != cudaSuccess)
            return CCE_ELAUNCH;
        }
        if (cudaStreamWaitEvent(st, side->ready[chunk & 1], 0) != cudaSuccess) return CCE_ELAUNCH;
      } else if (int rc = gather(chunk, st)) {
        return rc;
      }
      const __nv_bfloat16* Eb = Ecb[side ? (chunk & 1) : 0];
      if (!make_map(&segK, Eb, D, cv, D, BK, BN)) return CCE_ELAUNCH;
      if (!make_map(&segMN, Eb, D, cv, D, 64, 64)) return CCE_ELAUNCH;
      if ((pair_g || kl_pair) &&
          !make_map(&segKhalf, Eb, D, cv, D, BK, kl_pair ? BN / 4 : BN / 2))
        return CCE_ELAUNCH;
      row0 = 0;
    } else {
      if (!make_map(&segK, sg.s[s].E, D, ns, D, BK, BN)) return CCE_ELAUNCH;
      if (!make_map(&segMN, sg.s[s].E, D, ns, D, 64, 64)) return CCE_ELAUNCH;
      if ((pair_g || kl_pair) &&
          !make_map(&segKhalf, sg.s[s].E, D, ns, D, BK, kl_pair ? BN / 4 : BN / 2))
        return CCE_ELAUNCH;
    }
      // step 1: G for this chunk, with its zero-slice masks
      uint32_t* dh_mask = masks + (size_t)(chunk & 1) * mask_stride;
      uint32_t* de_mask = dh_mask + (size_t)(pl.Npad / BM) * dh_words;
      // unfiltered calls keep no zero-slice masks (every K step is issued)
      gp.mask_clear = use_masks ? masks + (size_t)((chunk + 1) & 1) * mask_stride : nullptr;
      gp.mask_clear_words = (int)(mask_bytes_for(pl.Npad, Vc) / sizeof(uint32_t));
      gp.dh_mask = use_masks ? dh_mask : nullptr;
      gp.dh_words = dh_words;
      gp.de_mask = use_masks ? de_mask : nullptr;
      gp.de_words = pl.de_words;
      gp.mapB = segK;
      gp.b_row0 = row0;
      gp.chunk_valid = cv;
      gp.ct = (int)cdiv(cv, kl_pair ? BN / 2 : BN);
      if (pair_g || kl_pair) gp.mapBdual = segKhalf;
      gp.seg = s;
      gp.c0 = c0;
      gp.Vc = Vc;
      gp.nkb = nkbD;
      gp.n_valid = cp.n_valid;
      gp.lse2_c = cp.lse2_c;
      gp.dloss_c = cp.dloss_c;
      gp.tseg = cp.tseg;
      gp.tpos = cp.tpos;
      gp.eps_keep = eps_keep;
      gp.l2eps = eps_keep > 0.f ? log2f(eps_keep) : -INFINITY;
      gp.G = G;
      gp.debug_keep = debug_keep;
      gp.debug_rows = (int)debug_rows;
      gp.words_per_row = words;
      gp.idx = cp.idx;
      gp.seg_begin = table.s[s].begin;
      gp.perm_seg = perm_seg;
      gp.status = status;
      gp.nz_list = sparse ? lists + (size_t)chunk * cap : nullptr;
      gp.nz_cnt = nz_cnt + chunk;
      gp.nz_cap = cap;
      gp.prev_nz_cnt = chunk > 0 ? nz_cnt + chunk - 1 : nullptr;
      gp.slab_flag = slab_flag + chunk;
      gp.repair = 0;
      gp.G_full = G_full;
      gp.tile_cmax2 = tile_skip ? tile_cmax2 + tile_off[s] + c0 / BN : nullptr;
      gp.blk_lse2min = blk_lse2min;
      gp.skip_l2 = gp.l2eps - 1.0f / 16.0f;  // margin over fp32 differences of the two logits
      const int g_grid = (int)std::min<int64_t>(sms, (int64_t)mbs * gp.ct);
      const int g_pairs = (int)std::min<int64_t>(sms / 2, cdiv(mbs, 2) * gp.ct);
      auto launch_g = [&]() {
        if (kl_pair) return launch_tc_pair<GPolicyKLPair>(gp, g_pairs, st, KC_G);
        if (kl) return launch_tc<GPolicyKL>(gp, g_grid, st, KC_G);
        if (full_de)
          return pair_g ? launch_tc_pair<GPolicyFullPair>(gp, g_pairs, st, KC_G)
                        : launch_tc<GPolicyFull>(gp, g_grid, st, KC_G);
        return pair_g ? launch_tc_pair<GPolicyPair>(gp, g_pairs, st, KC_G)
                      : launch_tc<GPolicy>(gp, g_grid, st, KC_G);
      };
      if (int rc = launch_g()) return rc;
      if (sparse) {  // recompute with the dense fallback if the chunk was mispredicted
        gp.repair = 1;
        if (int rc = launch_g()) return rc;
      }
      // step 2: dE rows of this chunk (chunks on the sparse route: after the loop)
      ep.nz_cnt = sparse_de ? nz_cnt + chunk : nullptr;
      ep.nz_cap = cap;
      ep.chunk_valid = cv;
      ep.mt = (int)cdiv(cv, pair_dedh ? 2 * BM : BM);
      ep.dt = dt;
      ep.D = (int)D;
      ep.c0 = c0;
      ep.perm_seg = perm_seg;
      ep.dE = sg.s[s].dE;
      ep.dE_comp = static_cast<__nv_bfloat16*>(sg.s[s].dE_comp);
      ep.mode = kahan ? 2 : (fp32 ? 1 : 0);
      ep.mask = use_masks ? de_mask : nullptr;
      ep.mwords = pl.de_words;
      ep.n_valid = cp.n_valid;
      ep.status = status;
      int de_rc;
      if (pair_dedh) {
        de_rc = launch_tc_pair<DEPairPolicy>(
            ep, (int)std::min<int64_t>(sms / 2, (int64_t)ep.mt * dt), st, KC_DE);
      } else {
        de_rc = launch_tc<DEPolicy>(ep, (int)std::min<int64_t>(sms, (int64_t)ep.mt * dt), st, KC_DE);
      }
      if (de_rc) return de_rc;
      // step 3: dH += G E_chunk
      hp.mapB = segMN;
      hp.b_row0 = row0;
      hp.nkb = (int)cdiv(cv, BK);
      hp.dt = dt;
      hp.D = (int)D;
      hp.dH_acc = dH_acc;
      hp.nz_cnt = sparse ? nz_cnt + chunk : nullptr;
      hp.nz_cap = cap;
      hp.mask = use_masks ? dh_mask : nullptr;
      hp.mwords = dh_words;
      hp.mblocks = mbs;
      hp.n_valid = cp.n_valid;
      hp.status = status;
      if (int rc = pair_dedh
                       ? launch_tc_pair<DHPairPolicy>(
                             hp, (int)std::min<int64_t>(sms / 2, cdiv(mbs, 2) * dt), st, KC_DH)
                       : launch_tc<DHPolicy>(hp, (int)std::min<int64_t>(sms, (int64_t)mbs * dt), st,
                                             KC_DH))
        return rc;
      if (side && cudaEventRecord(side->freed[chunk & 1], st) != cudaSuccess) return CCE_ELAUNCH;
      return CCE_OK;
  };
  int loop_rc = CCE_OK;
  for (int k = 0; k < n_chunks && loop_rc == CCE_OK; ++k) loop_rc = do_chunk(k);
  if (side) {  // join the side stream back into the caller's stream
    const bool ok = cudaEventRecord(side->join, side->ss) == cudaSuccess &&
                    cudaStreamWaitEvent(st, side->join, 0) == cudaSuccess;
    if (loop_rc == CCE_OK && !ok) loop_rc = CCE_ELAUNCH;
  }
  if (loop_rc != CCE_OK) return loop_rc;
  const int chunk = n_chunks;
  // sparse chunks: lists -> CSR by column (dE) and by row (dH), then the gathers
  const int gthreads = gather_threads(D);
  const int gblocks = sms * std::max(1, 2048 / gthreads);
  if (sparse) {
    if (cudaMemsetAsync(row_cnt, 0, sizeof(int) * (size_t)(pl.Npad + 1), st) != cudaSuccess ||
        (sparse_de && cudaMemsetAsync(col_cnt, 0, sizeof(int) * (size_t)(v_live + 1), st) != cudaSuccess))
      return CCE_ELAUNCH;
    SparseListParams lp;
    lp.nz_cnt = nz_cnt;
    lp.nch = chunk;
    lp.cap = cap;
    lp.lists = lists;
    lp.cmap = cmap;
    lp.col_cnt = sparse_de ? col_cnt : nullptr;
    lp.col_ptr = col_ptr;
    lp.csorted = csorted;
    lp.row_cnt = row_cnt;
    lp.row_ptr = row_ptr;
    lp.rsorted = rsorted;
    const dim3 lgrid((unsigned)std::min<int64_t>(cdiv(cap, 256), std::max(1, 4 * sms / chunk)), chunk);
    {
      TimedLaunch tl_(KC_SPARSE, st);
      sparse_count_kernel<<<lgrid, 256, 0, st>>>(lp);
    }
    if (launched()) return CCE_ELAUNCH;
    void* scan_tmp = at<void>(workspace, pl.off_scan);
    for (int pass = 0; pass < 2; ++pass) {
      if (pass == 0 && !sparse_de) continue;
      int* cnt = pass == 0 ? col_cnt : row_cnt;
      int* ptr = pass == 0 ? col_ptr : row_ptr;
      const int n = (int)(pass == 0 ? v_live + 1 : pl.Npad + 1);
      size_t need = 0;
      if (cub::DeviceScan::ExclusiveSum(nullptr, need, cnt, ptr, n, st) != cudaSuccess ||
          need > pl.scan_bytes)
        return CCE_ELAUNCH;
      TimedLaunch tl_(KC_SPARSE, st);
      if (cub::DeviceScan::ExclusiveSum(scan_tmp, need, cnt, ptr, n, st) != cudaSuccess)
        return CCE_ELAUNCH;
    }
    {
      TimedLaunch tl_(KC_SPARSE, st);
      sparse_scatter_kernel<<<lgrid, 256, 0, st>>>(lp);
    }
    if (launched()) return CCE_ELAUNCH;
    if (sparse_de) {
      DERows dr;
      memset(&dr, 0, sizeof(dr));
      dr.ptr = col_ptr;
      dr.ent = csorted;
      dr.Hc = Hc;
      dr.v_live = v_live;
      dr.D = (int)D;
      dr.range = gather_range(v_live, gblocks);
      dr.nz_cnt = nz_cnt;
      dr.cap = cap;
      dr.cmap = cmap;
      dr.vocab_perm = vocab_perm;
      for (int s = 0; s < sg.n; ++s) dr.dE[s] = sg.s[s].dE;
      dr.fp32_out = fp32 ? 1 : 0;
      {
        TimedLaunch tl_(KC_SPARSE, st);
        const int grid = (int)std::min<int64_t>(cdiv(v_live, dr.range), gblocks);
        if (fp32)
          csr_rows_kernel<DERows, true><<<grid, gthreads, 0, st>>>(dr);
        else
          csr_rows_kernel<DERows, false><<<grid, gthreads, 0, st>>>(dr);
      }
      if (launched()) return CCE_ELAUNCH;
    }
  }
  DHRows hr;
  memset(&hr, 0, sizeof(hr));
  hr.ptr = sparse ? row_ptr : nullptr;
  hr.ent = rsorted;
  hr.n_valid = cp.n_valid;
  hr.idx = cp.idx;
  hr.dH_acc = dH_acc;
  hr.nz_cnt = sparse ? nz_cnt : nullptr;
  hr.nch = chunk;
  hr.cap = cap;
  hr.D = (int)D;
  hr.range = gather_range(pl.Npad, gblocks);
  hr.dH = dH;
  hr.fp32_out = fp32_dh ? 1 : 0;
  for (int s = 0; s < sg.n; ++s) {
    hr.E[s] = table.s[s].E;
    hr.live_off[s] = table.s[s].live_off;
  }
  hr.vocab_perm = vocab_perm;
  {
    TimedLaunch tl_(KC_SPARSE, st);
    const int grid = (int)std::min<int64_t>(cdiv(pl.Npad, hr.range), gblocks);
    if (fp32_dh)
      csr_rows_kernel<DHRows, true><<<grid, gthreads, 0, st>>>(hr);
    else
      csr_rows_kernel<DHRows, false><<<grid, gthreads, 0, st>>>(hr);
  }
  if (launched()) return CCE_ELAUNCH;
  {
    TimedLaunch tl_(KC_SPARSE, st);
    dh_fill_kernel<<<(int)std::min<int64_t>(cdiv(N * (D / 8), 256), sms * 8), 256, 0, st>>>(
        cp.pos_of_row, N, (int)D, dH, fp32_dh ? 1 : 0);
  }
  return launched();
}

}  // namespace

extern "C" {

int cce_bwd(const void* H, const void* E, const int32_t* y, const float* lse, const float* dloss,
            int64_t N, int64_t D, int64_t V, int32_t ignore_index, const cce_segment* segs,
            int32_t n_segs, float filter_eps, const int32_t* vocab_perm, const float* colmax,
            uint32_t flags, void* dH, void* dE, void* dE_comp, uint32_t* debug_keep,
            int64_t debug_rows, void* workspace, size_t workspace_bytes, int32_t* status,
            void* stream) {
  return bwd_impl(H, E, y, lse, dloss, N, D, V, ignore_index, segs, n_segs, filter_eps, vocab_perm,
                  colmax, flags, dH, dE, dE_comp, debug_keep, debug_rows, workspace,
                  workspace_bytes, status, stream, nullptr);
}

// ------------------------------------------------------------ soft-target KL
size_t cce_kl_fwd_workspace_size(int64_t N, int64_t D, int64_t V) {
  if (!sizes_ok(N, D, V)) return 0;
  return plan_kl_fwd(N, D, V).total;
}

int cce_kl_fwd(const void* Hs, const void* Es, const void* Ht, const void* Et,
               const int32_t* row_mask, int64_t N, int64_t D, int64_t V, float* kl, float* lse_s,
               float* lse_t, void* workspace, size_t workspace_bytes, int32_t* status,
               void* stream) {
  if (!sizes_ok(N, D, V)) return CCE_EINVAL;
  if (N == 0) return CCE_OK;
  if (!Hs || !Es || !Ht || !Et || !kl || !lse_s || !lse_t || !status || !aligned16(Hs) ||
      !aligned16(Es) || !aligned16(Ht) || !aligned16(Et))
    return CCE_EINVAL;
  const KLFwdPlan pl = plan_kl_fwd(N, D, V);
  if (!workspace || workspace_bytes < pl.total) return CCE_EWORKSPACE;
  const int sms = device_sms();
  if (sms <= 0 || !encode_fn()) return CCE_EDEVICE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  CompactParams cp;
  memset(&cp, 0, sizeof(cp));
  cp.y = row_mask;
  cp.N = (int)N;
  cp.ignore_index = 0;
  cp.no_target = 1;
  cp.idx = at<int>(workspace, pl.off_idx);
  cp.pos_of_row = at<int>(workspace, pl.off_pos);
  cp.n_valid = at<int>(workspace, pl.off_nvalid);
  cp.status = status;
  __nv_bfloat16* Hs_c = at<__nv_bfloat16>(workspace, pl.off_hs);
  __nv_bfloat16* Ht_c = at<__nv_bfloat16>(workspace, pl.off_ht);
  if (int rc = run_compaction(cp, Hs, pl.Npad, D, sms, Hs_c, st)) return rc;
  {
    TimedLaunch tl_(KC_AUX, st);
    gather_rows_kernel<<<sms * 4, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(Ht), cp.idx,
                                                cp.n_valid, (int)pl.Npad, (int)D, Ht_c);
  }
  if (launched()) return CCE_ELAUNCH;

  KLFwdParams kp;
  memset(&kp, 0, sizeof(kp));
  if (!make_map(&kp.mapAs, Hs_c, D, pl.Npad, D, BK, BM) ||
      !make_map(&kp.mapAt, Ht_c, D, pl.Npad, D, BK, BM) ||
      !make_map(&kp.mapBs, Es, D, V, D, BK, BN) || !make_map(&kp.mapBt, Et, D, V, D, BK, BN))
    return CCE_ELAUNCH;
  kp.V = (int)V;
  kp.T_v = pl.T_v;
  kp.tpi = pl.tpi;
  kp.S = pl.S;
  kp.Npad = (int)pl.Npad;
  kp.nkb = (int)cdiv(D, BK);
  kp.n_valid = cp.n_valid;
  kp.part = at<float>(workspace, pl.off_part);
  kp.status = status;
  // (single CTAs: on CTA pairs this forward ran 1.5% faster, but the
  // backward kernels after it ran up to 4.5% slower under the power cap)
  const int64_t items = (pl.Npad / BM) * pl.S;
  if (int rc = launch_tc<KLFwdPolicy>(kp, (int)std::min<int64_t>(sms, items), st, KC_FWD)) return rc;
  KLFinParams fin;
  fin.pos_of_row = cp.pos_of_row;
  fin.part = kp.part;
  fin.N = (int)N;
  fin.S = pl.S * kKLFwdHalves;
  fin.Npad = (int)pl.Npad;
  fin.kl = kl;
  fin.lse_s = lse_s;
  fin.lse_t = lse_t;
  {
    TimedLaunch tl_(KC_AUX, st);
    kl_finalize_kernel<<<(int)std::min<int64_t>(cdiv(N, 8), sms * 8), 256, 0, st>>>(fin);
  }
  return launched();
}

size_t cce_kl_bwd_workspace_size(int64_t N, int64_t D, int64_t V, uint32_t flags) {
  if (!sizes_ok(N, D, V)) return 0;
  return plan_bwd(N, D, V, flags, true).total;
}

int cce_kl_bwd(const void* Hs, const void* Es, const void* Ht, const void* Et,
               const int32_t* row_mask, const float* lse_s, const float* lse_t,
               const float* dloss, int64_t N, int64_t D, int64_t V, float filter_eps,
               uint32_t flags, void* dH, void* dE, void* dE_comp, uint32_t* debug_keep,
               int64_t debug_rows, void* workspace, size_t workspace_bytes, int32_t* status,
               void* stream) {
  const KLArgs a{Ht, Et, lse_t};
  return bwd_impl(Hs, Es, row_mask, lse_s, dloss, N, D, V, 0, nullptr, 0, filter_eps, nullptr,
                  nullptr, flags, dH, dE, dE_comp, debug_keep, debug_rows, workspace,
                  workspace_bytes, status, stream, &a);
}


size_t cce_vocab_sort_workspace_size(int64_t N, int64_t V, int32_t n_segs) {
  (void)N;
  if (V <= 0 || V > (int64_t)INT32_MAX - 256 || n_segs < 0 || n_segs > CCE_MAX_SEGMENTS) return 0;
  return plan_sort(V).total;
}

int cce_vocab_sort(const float* colmax, const int32_t* y, int64_t N, int64_t V, int32_t ignore_index,
                   const cce_segment* segs, int32_t n_segs, int32_t* vocab_perm, void* workspace,
                   size_t workspace_bytes, void* stream) {
  if (V <= 0 || N < 0 || !vocab_perm) return CCE_EINVAL;
  if (!colmax && !y && N > 0) return CCE_EINVAL;
  Segs sg;
  // the classifier pointers are not needed here; accept any non-null marker
  if (segs == nullptr || n_segs == 0) {
    sg.n = 1;
    sg.s[0] = cce_segment{0, V, vocab_perm, nullptr, nullptr};
    sg.live = V;
  } else {
    cce_segment tmp[CCE_MAX_SEGMENTS];
    if (n_segs < 0 || n_segs > CCE_MAX_SEGMENTS) return CCE_EINVAL;
    for (int i = 0; i < n_segs; ++i) {
      tmp[i] = segs[i];
      tmp[i].E = vocab_perm;
    }
    if (int rc = build_segs(nullptr, V, tmp, n_segs, sg)) return rc;
  }
  const SortPlan pl = plan_sort(V);
  if (!workspace || workspace_bytes < pl.total) return CCE_EWORKSPACE;
  const int sms = device_sms();
  if (sms <= 0) return CCE_EDEVICE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int T_v = 0;
  const SegTable table = dev_table(sg, &T_v);
  float* key = at<float>(workspace, pl.off_key);
  float* key_out = at<float>(workspace, pl.off_key_out);
  int* ids = at<int>(workspace, pl.off_ids);
  void* tmp = at<void>(workspace, pl.off_tmp);
  if (colmax) {
    if (cudaMemcpyAsync(key, colmax, sizeof(float) * sg.live, cudaMemcpyDeviceToDevice, st) !=
        cudaSuccess)
      return CCE_ELAUNCH;
  } else {
    if (cudaMemsetAsync(key, 0, sizeof(float) * sg.live, st) != cudaSuccess) return CCE_ELAUNCH;
    if (N > 0) {
      target_hist_kernel<<<sms * 4, 256, 0, st>>>(y, (int)N, ignore_index, table, key);
      if (launched()) return CCE_ELAUNCH;
    }
  }
  for (int s = 0; s < sg.n; ++s) {
    const int n = table.s[s].n, off = table.s[s].live_off;
    iota_kernel<<<(int)std::min<int64_t>(cdiv(n, 256), sms * 8), 256, 0, st>>>(ids + off, n);
    if (launched()) return CCE_ELAUNCH;
    size_t need = 0;
    if (cub::DeviceRadixSort::SortPairsDescending(nullptr, need, key + off, key_out + off, ids + off,
                                                  vocab_perm + off, n, 0, 32, st) != cudaSuccess)
      return CCE_ELAUNCH;
    if (need > pl.tmp_bytes) return CCE_EWORKSPACE;
    size_t have = pl.tmp_bytes;
    if (cub::DeviceRadixSort::SortPairsDescending(tmp, have, key + off, key_out + off, ids + off,
                                                  vocab_perm + off, n, 0, 32, st) != cudaSuccess)
      return CCE_ELAUNCH;
    if (launched()) return CCE_ELAUNCH;  // counted as one (a short sequence of cub kernels)
  }
  return CCE_OK;
}

int cce_vocab_combine(const float* parts, int32_t R, const int32_t* y, int64_t N, int64_t V,
                      int32_t ignore_index, const cce_segment* segs, int32_t n_segs, float* loss,
                      float* lse, void* stream) {
  if (N < 0 || N > (int64_t)INT32_MAX || R < 1 || R > 4096 || V <= 0) return CCE_EINVAL;
  // only the head's logical ranges matter here: validate them with a stand-in
  // classifier pointer
  Segs sg;
  if (segs == nullptr || n_segs == 0) {
    sg.n = 1;
    sg.s[0] = cce_segment{0, V, parts, nullptr, nullptr};
  } else {
    if (n_segs < 0 || n_segs > CCE_MAX_SEGMENTS) return CCE_EINVAL;
    cce_segment tmp[CCE_MAX_SEGMENTS];
    for (int i = 0; i < n_segs; ++i) {
      tmp[i] = segs[i];
      tmp[i].E = parts;
    }
    if (build_segs(nullptr, V, tmp, n_segs, sg) != CCE_OK) return CCE_EINVAL;
  }
  if (N == 0) return CCE_OK;
  if (!parts || !y || !loss || !lse) return CCE_EINVAL;
  const int sms = device_sms();
  if (sms <= 0) return CCE_EDEVICE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const SegTable table = dev_table(sg, nullptr);
  {
    TimedLaunch tl_(KC_AUX, st);
    vocab_combine_kernel<<<(int)std::min<int64_t>(cdiv(N, 256), sms * 8), 256, 0, st>>>(
        parts, R, y, (int)N, ignore_index, table, V, loss, lse);
  }
  return launched();
}

int cce_debug_stall(uint64_t wait_ns, int32_t* status, void* stream) {
  if (!status || wait_ns == 0 || wait_ns > 1000000000ull) return CCE_EINVAL;
  if (device_sms() <= 0) return CCE_EDEVICE;
  StallParams sp;
  sp.status = status;
  sp.wait_ns = wait_ns;
  return launch_tc<StallPolicy>(sp, 1, static_cast<cudaStream_t>(stream), KC_AUX);
}

int cce_debug_stall_pair(uint64_t wait_ns, int32_t* status, void* stream) {
  if (!status || wait_ns == 0 || wait_ns > 1000000000ull) return CCE_EINVAL;
  if (device_sms() <= 0) return CCE_EDEVICE;
  StallParams sp;
  sp.status = status;
  sp.wait_ns = wait_ns;
  return launch_tc_pair<StallPairPolicy>(sp, 1, static_cast<cudaStream_t>(stream), KC_AUX);
}

uint64_t cce_launch_count(void) { return g_launches.load(); }

int cce_timing_enable(uint32_t class_mask) {
  if (class_mask >= (1u << KC_N)) return CCE_EINVAL;
  g_timing.mask = class_mask;
  return CCE_OK;
}

int cce_timing_read(float* ms, int64_t* launches, int32_t n_classes) {
  if (!ms || !launches || n_classes < 0 || n_classes > KC_N) return CCE_EINVAL;
  for (int c = 0; c < n_classes; ++c) {
    ms[c] = 0.f;
    launches[c] = 0;
  }
  int rc = CCE_OK;
  for (const auto& r : g_timing.rec) {
    float t = 0.f;
    if (cudaEventSynchronize(g_timing.pool[r.second + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&t, g_timing.pool[r.second], g_timing.pool[r.second + 1]) != cudaSuccess) {
      rc = CCE_ELAUNCH;
      continue;
    }
    if (r.first < n_classes) {
      ms[r.first] += t;
      launches[r.first] += 1;
    }
  }
  g_timing.rec.clear();
  g_timing.used = 0;
  return rc;
}

}  // extern "C"
