// Per-16-wide-input-block Hessian accumulation (raw sums).
//
// Method: "add local hessian calibration" (PR #788), Overview (H_n = X_b^T X_b per block);
// "Add activation-aware local Hessian scale calibration" (PR #1976), "What does this PR do?"
// (H = X_q^T X_q, P = X_q^T (X_q - X)); "Add WMSE weight scale search calibration" (PR #2283),
// "How" (Imp = column sums of squares in a [n_blocks, 16] buffer); "[2/3] Speed up layerwise
// GPTQ on MoE models" (PR #2864), embedded #2840 (one Hessian per expert over its routed tokens).
//
// Kernels (all HBM-bound):
//  * accum_mma_kernel: bf16 FULL / ACT on tensor cores. A CTA owns a 128-column slab (8
//    blocks, one per warp) and a token range; 64-token x 128-column tiles stream through a
//    4-stage (FULL) or 3-stage (ACT) cp.async ring in XOR-swizzled shared memory. Each warp
//    turns 16 tokens of its block into one ldmatrix.x4.trans, which is at once the A fragment
//    (X_b^T) and both B fragments (X_b) of two m16n8k16 MMAs: the 16x16 block Hessian with no
//    wasted MACs. bf16 x bf16 products are exact in the fp32 accumulator. For P the
//    difference D = X_q - X (exact in fp32) is split into bf16 hi + lo parts, two more MMAs
//    each. (Forming P as H - X_q^T X instead would cost two MMAs fewer, but the cancellation
//    multiplies the accumulation error by |H| / |P|, which exceeds 100 on real blocks.)
//    Dense layers with enough slabs to fill a wave: clusters of up to 8 CTAs split a slab's
//    tokens and reduce in distributed shared memory. Narrower dense layers: token splits write
//    partials to the workspace, which reduce_partials_kernel sums in a fixed order. Grouped
//    (MoE): a persistent grid deals the (slab, expert) pairs round-robin in slab-major order, so
//    that the CTAs in flight share one or two slabs of X in L2; a CTA runs one pipeline through
//    its pairs, gathering the routed rows through the CSR, and writes each expert's sums after
//    its last tile.
//    Activation-aware with the input quantizer fused (QUANT): only X streams in; each warp
//    turns its block's 64 x 16 slice of the tile into X_q in shared memory (act_quant.cuh)
//    and synchronises only with itself before the MMAs, so X is read from HBM once.
//  * accum_diag_kernel: bf16 DIAG column sums of squares; each thread streams 8 columns
//    (16-byte loads) over a token range; partials to the workspace, then reduce.
//  * accum_generic_kernel: CUDA-core fp32 path for fp32 inputs (and grouped bf16 DIAG).
#include <cooperative_groups.h>

#include "act_quant.cuh"
#include "common.cuh"

namespace lhcal {
namespace {

// ---------------------------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // 0 source bytes: the 16 destination bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }

__device__ __forceinline__ void lds128(uint32_t addr, uint32_t* v) {
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
               : "r"(addr));
}

__device__ __forceinline__ void sts128(uint32_t addr, const uint32_t* v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(addr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3])
               : "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                                  uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D += A (16x16 bf16, row) * B (16x8 bf16, col), fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// bf16x2 (as uint32) -> two floats, exact.
__device__ __forceinline__ float2 bf2_to_f2(uint32_t v) {
  return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}

__device__ __forceinline__ uint32_t f2_to_bf2(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

// D = Xq - X for a bf16x2 pair, split into bf16 hi + lo (hi + lo = D to ~2^-17 relative). Both
// differences are exact in fp32; packed fp32 FMAs (x * -1 + y) do the pair at once.
__device__ __forceinline__ void diff_split(uint32_t xq, uint32_t x, uint32_t& hi, uint32_t& lo) {
  const float2 m1 = make_float2(-1.f, -1.f);
  const float2 d = __ffma2_rn(bf2_to_f2(x), m1, bf2_to_f2(xq));
  hi = f2_to_bf2(d.x, d.y);
  const float2 r = __ffma2_rn(bf2_to_f2(hi), m1, d);
  lo = f2_to_bf2(r.x, r.y);
}

// ---------------------------------------------------------------------------------------------
// Tensor-core FULL / ACT accumulation
// ---------------------------------------------------------------------------------------------

constexpr int kMmaThreads = 256;  // 8 warps
constexpr int kSlabCols = 128;    // 8 blocks of 16 columns
constexpr int kTileTok = 64;
constexpr int kRowBytes = kSlabCols * 2;              // 256 B per token row of the slab
constexpr int kTileBytes = kTileTok * kRowBytes;      // 16 KB per tensor per stage
constexpr int64_t kMaxStagedItems = 1024;             // grouped items per CTA (16 KB of item records)

// Shared memory: the cp.async ring (X_q and X per stage for ACT, X for FULL and QUANT), the
// token-id ring, and for QUANT the X_q tile the warps write plus the quantizer tables.
template <bool ACT, bool QUANT>
struct MmaCfg {
  static constexpr bool kTwo = ACT && !QUANT;  // two tensors stream in
  static constexpr int kStages = ACT ? 3 : 4;
  // Resident CTAs per SM the launch plans for: FULL 65 KB and QUANT 74 KB of shared memory
  // fit three, ACT's 97 KB two.
  static constexpr int kResident = kTwo ? 2 : 3;
  // Clusters (cs <= 8 CTAs per slab) are used when they fill at least this fraction of a wave
  // of resident CTAs; otherwise token splits and a reduction. The fused quantizer is bound by
  // its integer pipe and wants every resident warp; the streaming variants are bound by HBM.
  static constexpr double kClusterFill = QUANT ? 0.9 : 0.5;
  static constexpr int kRing = kStages * (kTwo ? 2 : 1) * kTileBytes;
  static constexpr int kIds = kStages * kTileTok * 4;
  static constexpr int kXq = QUANT ? kTileBytes : 0;
  static constexpr int kTab = QUANT ? static_cast<int>(sizeof(ActQuantTables)) : 0;
  static constexpr int kSmem = kRing + kIds + kXq + kTab;
};

// Byte offset of 16-byte chunk c (0..15) of tile row r in the swizzled layout.
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return static_cast<uint32_t>(r * kRowBytes + ((c ^ (r & 7)) << 4));
}

constexpr uint32_t kBand = 16 * kRowBytes;  // 16 rows: the swizzle repeats every 8


__device__ __forceinline__ void cp_async16_all(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}

// What a thread copies of each tile: row r = tid / 4 and its 16-byte chunks c = j + 4 m (j = tid
// % 4, m = 0..3), so that four lanes cover 64 contiguous bytes of the row per copy and the
// thread needs one row address per tile (the chunks are 64 bytes apart). With x = r & 7, the
// swizzled chunk c ^ x sits at byte 16 (j ^ (x & 3)) + 64 ((m & 1) ^ (x >> 2)) + 128 (m >> 1) of
// the row: d0 for even m, d1 for odd m, plus 128 for m >= 2.
struct TileRow {
  uint32_t d0, d1;  // swizzled byte offsets of chunks m = 0 and m = 1 in a stage
  int r;            // tile row
  int j;            // first chunk
};

__device__ __forceinline__ TileRow tile_row(int tid) {
  TileRow t;
  t.r = tid >> 2;
  t.j = tid & 3;
  const int x = t.r & 7;
  const uint32_t base = static_cast<uint32_t>(t.r * kRowBytes + 16 * (t.j ^ (x & 3)));
  t.d0 = base + 64 * (x >> 2);
  t.d1 = base + 64 * (1 - (x >> 2));
  return t;
}

// Loads one 64-token x 128-column tile (both tensors for ACT) into the stage at shared address
// stage: rows pos0 + r with pos0 + r < end, the row of position pos0 + r being ids_s[r] (grouped;
// shared memory) or the position itself (dense). col is the thread's first element in a row (the
// slab's first column + 8 j); bit m of cmask says whether chunk m lies inside cin. Rows past end
// and chunks past cin are zero-filled.
template <bool TWO>
__device__ __forceinline__ void load_tile(uint32_t stage, const TileRow& tr, const __nv_bfloat16* x,
                                          const __nv_bfloat16* xq, int64_t ldx, int64_t col, uint32_t cmask,
                                          const int32_t* ids_s, int64_t pos0, int64_t end) {
  const bool row_ok = pos0 + tr.r < end;
  const int64_t row = ids_s ? static_cast<int64_t>(ids_s[tr.r]) : pos0 + tr.r;
  if (row_ok && cmask == 0xfu) {
    const int64_t off = row * ldx + col;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const uint32_t dst = stage + ((m & 1) ? tr.d1 : tr.d0) + 128 * (m >> 1);
      if (TWO) {
        cp_async16_all(dst, xq + off + 32 * m);
        cp_async16_all(dst + kTileBytes, x + off + 32 * m);
      } else {
        cp_async16_all(dst, x + off + 32 * m);
      }
    }
    return;
  }
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const bool ok = row_ok && ((cmask >> m) & 1u);
    const int64_t off = ok ? row * ldx + col + 32 * m : 0;
    const uint32_t dst = stage + ((m & 1) ? tr.d1 : tr.d0) + 128 * (m >> 1);
    if (TWO) {
      cp_async16(dst, xq + off, ok);
      cp_async16(dst + kTileBytes, x + off, ok);
    } else {
      cp_async16(dst, x + off, ok);
    }
  }
}

// Copies the 64 token ids of the tile at positions [pos0, pos0 + 64) (zeros past end) into a
// shared-memory slot with cp.async; 16 threads move 16 bytes each.
__device__ __forceinline__ void load_ids(int32_t* slot, const int32_t* ids, int64_t pos0, int64_t end) {
  const int tid = threadIdx.x;
  if (tid < kTileTok / 4) {
    const int64_t pos = pos0 + 4 * tid;
    const uint32_t dst = smem_u32(slot + 4 * tid);
    if (pos + 4 <= end && ((reinterpret_cast<uintptr_t>(ids + pos) & 15) == 0)) {
      cp_async16(dst, ids + pos, true);
    } else {
      // Ragged or unaligned: element by element (4-byte copies), zeros past end.
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const bool ok = pos + j < end;
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(dst + 4 * j),
                     "l"(ids + (ok ? pos + j : 0)), "r"(ok ? 4 : 0));
      }
    }
  }
}

// A CTA works through a list of items, each a (128-column slab, row set) pair. Dense: one item,
// slab blockIdx.x and token range blockIdx.y (a split, whose sums go to the workspace at
// split * out_item_stride). Grouped: the (slab, expert) pairs in slab-major order q = slab *
// groups + expert, dealt round-robin over the persistent grid (CTA c takes q = c, c + gridDim.x,
// ...), each summed over the expert's routed rows and written at expert * out_item_stride. The
// CTAs of a wave therefore work on one or two slabs at a time, whose rows (4 MB per slab) stay
// in L2 while the experts gather them. A single cp.async pipeline runs through the tiles of all
// items, so short items (about 5 tiles per expert) still stream; the accumulators are written
// out after each item's last tile. accumulate_into: out += sums. QUANT (with ACT): xq is unused
// and X_q comes from X through the input quantizer with the global scale *act_gx.
template <bool ACT, bool QUANT, bool CLUSTER>
__global__ void __launch_bounds__(kMmaThreads, QUANT ? 3 : 1)
accum_mma_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ xq,
                 int64_t tokens, int64_t cin, int64_t ldx, const int32_t* __restrict__ group_offsets,
                 const int32_t* __restrict__ token_ids, int64_t tok_per_split, int64_t total_items,
                 int64_t groups, float* __restrict__ out_h, float* __restrict__ out_p,
                 int64_t out_item_stride, int accumulate_into, const float* __restrict__ act_gx) {
  static_assert(ACT || !QUANT, "the input quantizer belongs to the activation-aware mode");
  using Cfg = MmaCfg<ACT, QUANT>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nblk = cin / kBlock;
  const bool grouped = group_offsets != nullptr;

  // This CTA's items are it0 <= item < it1. Grouped: item t is the pair q = blockIdx.x + t *
  // gridDim.x; dense: the one item blockIdx.y (the token split) of slab blockIdx.x.
  int64_t it0, it1;
  if (grouped) {
    it0 = 0;
    it1 = total_items > blockIdx.x ? ceil_div(total_items - blockIdx.x, gridDim.x) : 0;
  } else {
    it0 = blockIdx.y;
    it1 = it0 + 1;
  }
  // Pair indices fit in 32 bits: groups <= 65535 and slabs <= 65535 / 8 (checked by the API).
  const uint32_t ngroups = static_cast<uint32_t>(groups);
  // Grouped: each of this CTA's items as {first row position, end, slab, expert}, staged in
  // shared memory after the pipeline (every cursor looks them up at each item boundary; a
  // global load or a division there would stall the whole CTA).
  int4* items_s = reinterpret_cast<int4*>(smem + Cfg::kSmem);
  if (grouped) {
    for (int64_t t = threadIdx.x; t < it1; t += kMmaThreads) {
      const uint32_t q = blockIdx.x + static_cast<uint32_t>(t) * gridDim.x;
      const uint32_t ex = q % ngroups;
      items_s[t] = make_int4(__ldg(group_offsets + ex), __ldg(group_offsets + ex + 1), static_cast<int>(q / ngroups),
                             static_cast<int>(ex));
    }
    __syncthreads();
  }
  auto slab_of = [&](int64_t item) -> int64_t { return grouped ? items_s[item].z : blockIdx.x; };
  // Index of the item's sums in out (expert, or token split).
  auto out_of = [&](int64_t item) -> int64_t { return grouped ? items_s[item].w : item; };
  auto range = [&](int64_t item, int64_t& b, int64_t& e) {
    if (grouped) {
      const int4 r = items_s[item];
      b = r.x;
      e = r.y;
    } else {
      b = item * tok_per_split;
      e = imin64(tokens, b + tok_per_split);
    }
  };

  // Accumulator layout of m16n8: c0,c1 -> (i = lane/4, j = 2*(lane%4) + {0,1}); c2,c3 -> i + 8.
  // Sums are written with streaming stores: they are not read again by this launch and should
  // not displace the activation rows that other CTAs are still gathering from L2.
  const int i0 = lane >> 2, j0 = 2 * (lane & 3);
  auto write_out = [&](int64_t item, const float (&ah)[2][4], const float (&ap)[2][4]) {
    const int64_t blk = slab_of(item) * 8 + warp;
    if (blk >= nblk) return;
    float* oh = out_h + out_of(item) * out_item_stride + blk * 256;
    float* op = ACT ? out_p + out_of(item) * out_item_stride + blk * 256 : nullptr;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int idx = (i0 + 8 * half) * 16 + nt * 8 + j0;
        float2 vh = make_float2(ah[nt][2 * half], ah[nt][2 * half + 1]);
        if (accumulate_into) {
          const float2 o = *reinterpret_cast<const float2*>(oh + idx);
          vh.x += o.x;
          vh.y += o.y;
        }
        __stcs(reinterpret_cast<float2*>(oh + idx), vh);
        if (ACT) {
          float2 vp = make_float2(ap[nt][2 * half], ap[nt][2 * half + 1]);
          if (accumulate_into) {
            const float2 o = *reinterpret_cast<const float2*>(op + idx);
            vp.x += o.x;
            vp.y += o.y;
          }
          __stcs(reinterpret_cast<float2*>(op + idx), vp);
        }
      }
    }
  };

  float acc_h[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  float acc_p[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};

  // Tiles over all items; items without rows produce zeros (OVERWRITE) or nothing (ADD).
  int64_t ntiles = 0;
  for (int64_t item = it0; item < it1; ++item) {
    int64_t b, e;
    range(item, b, e);
    if (e > b) ntiles += ceil_div(e - b, kTileTok);
    else if (!accumulate_into && !CLUSTER) write_out(item, acc_h, acc_p);
  }

  // Cursors (item, position, end): ids of tiles 2S-2 ahead of consumption (grouped), data of
  // tiles S-1 ahead, and the tile being consumed.
  auto first_nonempty = [&](int64_t item, int64_t& pos, int64_t& end) -> int64_t {
    for (; item < it1; ++item) {
      int64_t b, e;
      range(item, b, e);
      if (e > b) {
        pos = b;
        end = e;
        return item;
      }
    }
    return it1;
  };
  constexpr int S = Cfg::kStages;
  constexpr int stage_bytes = Cfg::kRing / S;
  int32_t* ids_ring = reinterpret_cast<int32_t*>(smem + Cfg::kRing);  // S slots of 64 ids
  uint8_t* xq_tile = smem + Cfg::kRing + Cfg::kIds;
  ActQuantTables* tab = reinterpret_cast<ActQuantTables*>(smem + Cfg::kRing + Cfg::kIds + Cfg::kXq);
  float inv6gx = 0.f;
  bool steps = false;
  if (QUANT) {
    const float gx = __ldg(act_gx);
    build_act_tables(*tab, gx, threadIdx.x, kMmaThreads);
    inv6gx = 1.f / (6.f * gx);  // only a first guess of each block's scale code
    steps = act_quant_steps(gx);
    __syncthreads();
  }
  int64_t i_pos = 0, i_end = 0, p_pos = 0, p_end = 0, c_pos = 0, c_end = 0;
  int64_t i_item = first_nonempty(it0, i_pos, i_end);
  int64_t i_tile = 0;
  int64_t p_item = first_nonempty(it0, p_pos, p_end);
  int64_t c_item = first_nonempty(it0, c_pos, c_end);
  // Ring slots of the id cursor, the data cursor and the consumer: tile t lives in slot t % S,
  // kept as wrapping counters (S = 3 would otherwise be a 64-bit division per tile).
  int i_slot = 0, p_slot = 0, c_slot = 0;
  auto next_slot = [](int v) { return v + 1 == S ? 0 : v + 1; };
  const uint32_t ring = smem_u32(smem);
  const TileRow trow = tile_row(threadIdx.x);
  // The data cursor's slab: the thread's first element in a row, and which of its chunks lie
  // inside cin.
  int64_t p_col = 0;
  uint32_t p_cmask = 0;
  auto set_slab = [&]() {
    p_col = (p_item < it1 ? slab_of(p_item) : 0) * kSlabCols + 8 * trow.j;
    p_cmask = 0;
#pragma unroll
    for (int m = 0; m < 4; ++m) p_cmask |= (p_col + 32 * m < cin ? 1u : 0u) << m;
  };
  set_slab();
  auto issue_ids = [&]() {  // ids of tile i_tile into slot i_tile % S
    if (grouped && i_tile < ntiles) {
      load_ids(ids_ring + i_slot * kTileTok, token_ids, i_pos, i_end);
      i_pos += kTileTok;
      if (i_pos >= i_end) i_item = first_nonempty(i_item + 1, i_pos, i_end);
    }
    ++i_tile;
    i_slot = next_slot(i_slot);
  };
  auto produce = [&]() {  // data of the next tile into its stage
    load_tile<Cfg::kTwo>(ring + p_slot * stage_bytes, trow, x, xq, ldx, p_col, p_cmask,
                         grouped ? ids_ring + p_slot * kTileTok : nullptr, p_pos, p_end);
    p_slot = next_slot(p_slot);
    p_pos += kTileTok;
    if (p_pos >= p_end) {
      p_item = first_nonempty(p_item + 1, p_pos, p_end);
      set_slab();
    }
  };

  // Ids of the first S - 1 tiles, then the prologue: data of tiles 0..S-2 and ids S-1..2S-3.
  for (int s2 = 0; s2 < S - 1; ++s2) issue_ids();
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
#pragma unroll
  for (int s2 = 0; s2 < S - 1; ++s2) {
    __syncthreads();  // the id slot refilled below was read by every thread for tile s2 - 1
    issue_ids();
    if (s2 < ntiles) produce();
    cp_async_commit();
  }

  // ldmatrix.x4.trans addressing: lane -> (matrix mi = lane / 8, row rr = lane % 8);
  // matrices: (tok 0-7, cols 0-7), (tok 0-7, cols 8-15), (tok 8-15, cols 0-7), (tok 8-15, cols 8-15).
  // Rows ts * 16 + lrow agree in their low three bits, so the 16-token steps are whole bands.
  const int mi = lane >> 3, rr = lane & 7;
  const int lrow = ((mi >> 1) << 3) + rr;
  const int lchunk = 2 * warp + (mi & 1);
  const uint32_t loff = swz(lrow, lchunk);

  for (int64_t it = 0; it < ntiles; ++it) {
    cp_async_wait<S - 2>();
    __syncthreads();
    issue_ids();  // tile it + 2S - 2
    if (it + S - 1 < ntiles) produce();  // tile it + S - 1
    cp_async_commit();
    const uint32_t base = ring + c_slot * stage_bytes;
    c_slot = next_slot(c_slot);
    uint32_t qbase = base;               // X_q (ACT) or X (FULL)
    uint32_t xbase = base + kTileBytes;  // X (ACT)
    if (QUANT) {
      // This warp's block: tokens lane and lane + 32, chunks 2 warp and 2 warp + 1 of the tile.
      qbase = smem_u32(xq_tile);
      xbase = base;
      // Both rows' loads, then both codes, then both table look-ups: the two dependency
      // chains (row -> code -> thresholds) overlap.
      uint32_t xv[2][8], av[2][8];
      int code[2];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int r = lane + 32 * half;
        lds128(base + swz(r, 2 * warp), xv[half]);
        lds128(base + swz(r, 2 * warp + 1), xv[half] + 4);
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) code[half] = act_block_code(xv[half], av[half], inv6gx, *tab, steps);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int r = lane + 32 * half;
        uint32_t qv[8];
        act_block_apply(xv[half], av[half], code[half], qv, *tab, steps);
        sts128(qbase + swz(r, 2 * warp), qv);
        sts128(qbase + swz(r, 2 * warp + 1), qv + 4);
      }
      __syncwarp();  // the ldmatrix below reads rows written by the other lanes of this warp
    }
#pragma unroll
    for (int ts = 0; ts < kTileTok / 16; ++ts) {
      const uint32_t off = loff + ts * kBand;
      uint32_t q0, q1, q2, q3;
      ldmatrix_x4_trans(qbase + off, q0, q1, q2, q3);
      mma_bf16(acc_h[0], q0, q1, q2, q3, q0, q2);
      mma_bf16(acc_h[1], q0, q1, q2, q3, q1, q3);
      if (ACT) {
        uint32_t x0, x1, x2, x3;
        ldmatrix_x4_trans(xbase + off, x0, x1, x2, x3);
        uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
        diff_split(q0, x0, h0, l0);
        diff_split(q1, x1, h1, l1);
        diff_split(q2, x2, h2, l2);
        diff_split(q3, x3, h3, l3);
        mma_bf16(acc_p[0], q0, q1, q2, q3, h0, h2);
        mma_bf16(acc_p[0], q0, q1, q2, q3, l0, l2);
        mma_bf16(acc_p[1], q0, q1, q2, q3, h1, h3);
        mma_bf16(acc_p[1], q0, q1, q2, q3, l1, l3);
      }
    }
    c_pos += kTileTok;
    if (c_pos >= c_end) {  // last tile of the consumer's item: write its sums
      if (CLUSTER) break;  // a dense item is the CTA's only one; the cluster reduces below
      write_out(c_item, acc_h, acc_p);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc_h[nt][v] = acc_p[nt][v] = 0.f;
      c_item = first_nonempty(c_item + 1, c_pos, c_end);
    }
  }
  cp_async_wait<0>();

  if (CLUSTER) {
    // The CTAs of a cluster summed disjoint token ranges of the same slab (dense). Each stages
    // its sums in its own shared memory; CTA rank q then adds block q of every CTA of the
    // cluster in rank order (distributed shared memory) and writes it.
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    float* stage = reinterpret_cast<float*>(smem);  // [H: 8 blocks x 256][P: 8 blocks x 256]
    __syncthreads();
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int idx = (i0 + 8 * half) * 16 + nt * 8 + j0;
        stage[warp * 256 + idx] = acc_h[nt][2 * half];
        stage[warp * 256 + idx + 1] = acc_h[nt][2 * half + 1];
        if (ACT) {
          stage[2048 + warp * 256 + idx] = acc_p[nt][2 * half];
          stage[2048 + warp * 256 + idx + 1] = acc_p[nt][2 * half + 1];
        }
      }
    }
    cluster.sync();
    const int csize = static_cast<int>(cluster.num_blocks());
    const int rank = static_cast<int>(cluster.block_rank());
    for (int b = rank; b < 8; b += csize) {  // blocks of the slab this CTA finishes
      const int64_t ob = static_cast<int64_t>(blockIdx.x) * 8 + b;
      if (ob < nblk) {
        const int t = threadIdx.x;  // 256 threads: one entry of the 16 x 16 block each
        float vh = 0.f, vp = 0.f;
        for (int q = 0; q < csize; ++q) {
          const float* rs = cluster.map_shared_rank(stage, q);
          vh += rs[b * 256 + t];
          if (ACT) vp += rs[2048 + b * 256 + t];
        }
        float* oh = out_h + ob * 256 + t;
        *oh = accumulate_into ? *oh + vh : vh;
        if (ACT) {
          float* op = out_p + ob * 256 + t;
          *op = accumulate_into ? *op + vp : vp;
        }
      }
    }
    cluster.sync();  // keep this CTA's staged sums alive until every rank has read them
  }
}

// ---------------------------------------------------------------------------------------------
// bf16 DIAG accumulation (dense)
// ---------------------------------------------------------------------------------------------

constexpr int kDiagThreads = 256;
constexpr int kDiagCols = kDiagThreads * 8;  // 2048 columns per CTA
constexpr int kDiagUnroll = 8;

__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void sq_acc(float* acc, const uint4& v) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = bf2_to_f2(u[i]);
    acc[2 * i] = fmaf(f.x, f.x, acc[2 * i]);
    acc[2 * i + 1] = fmaf(f.y, f.y, acc[2 * i + 1]);
  }
}

__global__ void __launch_bounds__(kDiagThreads)
accum_diag_kernel(const __nv_bfloat16* __restrict__ x, int64_t tokens, int64_t cin, int64_t ldx,
                  int64_t tok_per_split, float* __restrict__ ws) {
  const int64_t col = static_cast<int64_t>(blockIdx.x) * kDiagCols + threadIdx.x * 8;
  if (col >= cin) return;
  const int64_t t0 = static_cast<int64_t>(blockIdx.y) * tok_per_split;
  const int64_t t1 = imin64(tokens, t0 + tok_per_split);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const __nv_bfloat16* p = x + t0 * ldx + col;
  int64_t t = t0;
  for (; t + kDiagUnroll <= t1; t += kDiagUnroll, p += kDiagUnroll * ldx) {
    uint4 v[kDiagUnroll];
#pragma unroll
    for (int u = 0; u < kDiagUnroll; ++u) v[u] = ld_stream16(p + u * ldx);
#pragma unroll
    for (int u = 0; u < kDiagUnroll; ++u) sq_acc(acc, v[u]);
  }
  for (; t < t1; ++t, p += ldx) sq_acc(acc, ld_stream16(p));
  float4* dst = reinterpret_cast<float4*>(ws + static_cast<int64_t>(blockIdx.y) * cin + col);
  dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

// ---------------------------------------------------------------------------------------------
// Generic CUDA-core accumulation (fp32 inputs; grouped bf16 DIAG)
// ---------------------------------------------------------------------------------------------

constexpr int kGenTok = 32;

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// One CTA of 256 threads per (block n, split or group). Thread (i, j) owns H_ij (and P_ij);
// DIAG uses threads 0..15. Partials / results go to out + (split or group) stride.
template <typename T, int MODE>
__global__ void __launch_bounds__(256)
accum_generic_kernel(const T* __restrict__ x, const T* __restrict__ xq, int64_t tokens, int64_t cin,
                     int64_t ldx, const int32_t* __restrict__ group_offsets,
                     const int32_t* __restrict__ token_ids, int64_t tok_per_split, float* __restrict__ out_h,
                     float* __restrict__ out_p, int64_t out_stride, int accumulate_into) {
  __shared__ float sx[kGenTok][kBlock];
  __shared__ float sq[kGenTok][kBlock];
  const int64_t n = blockIdx.x;
  const int tid = threadIdx.x, i = tid >> 4, j = tid & 15;
  int64_t b0, b1;
  const bool grouped = group_offsets != nullptr;
  if (grouped) {
    b0 = __ldg(group_offsets + blockIdx.y);
    b1 = __ldg(group_offsets + blockIdx.y + 1);
  } else {
    b0 = static_cast<int64_t>(blockIdx.y) * tok_per_split;
    b1 = imin64(tokens, b0 + tok_per_split);
  }
  float ah = 0.f, ap = 0.f;
  for (int64_t pos0 = b0; pos0 < b1; pos0 += kGenTok) {
    for (int e = tid; e < kGenTok * kBlock; e += 256) {
      const int tt = e >> 4, cc = e & 15;
      const int64_t pos = pos0 + tt;
      float vx = 0.f, vq = 0.f;
      if (pos < b1) {
        const int64_t row = grouped ? static_cast<int64_t>(__ldg(token_ids + pos)) : pos;
        const int64_t off = row * ldx + n * kBlock + cc;
        vx = to_f32<T>(x[off]);
        if (MODE == LHCAL_ACT_AWARE) vq = to_f32<T>(xq[off]);
      }
      sx[tt][cc] = vx;
      sq[tt][cc] = vq;
    }
    __syncthreads();
    if (MODE == LHCAL_DIAG) {
      if (tid < kBlock)
        for (int tt = 0; tt < kGenTok; ++tt) ah = fmaf(sx[tt][tid], sx[tt][tid], ah);
    } else if (MODE == LHCAL_FULL) {
      for (int tt = 0; tt < kGenTok; ++tt) ah = fmaf(sx[tt][i], sx[tt][j], ah);
    } else {
      for (int tt = 0; tt < kGenTok; ++tt) {
        ah = fmaf(sq[tt][i], sq[tt][j], ah);
        ap = fmaf(sq[tt][i], sq[tt][j] - sx[tt][j], ap);
      }
    }
    __syncthreads();
  }
  const int64_t base = static_cast<int64_t>(blockIdx.y) * out_stride;
  if (MODE == LHCAL_DIAG) {
    if (tid < kBlock) {
      float* o = out_h + base + n * kBlock + tid;
      *o = accumulate_into ? *o + ah : ah;
    }
  } else {
    float* o = out_h + base + n * 256 + tid;
    *o = accumulate_into ? *o + ah : ah;
    if (MODE == LHCAL_ACT_AWARE) {
      float* q = out_p + base + n * 256 + tid;
      *q = accumulate_into ? *q + ap : ap;
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Fixed-order reduction of split partials: out[i] (+)= sum_s ws[s * stride + i]
// ---------------------------------------------------------------------------------------------

__global__ void reduce_partials_kernel(const float* __restrict__ ws, int64_t splits, int64_t stride,
                                       int64_t count, float* __restrict__ out, int accumulate_into) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float s = 0.f;
    for (int64_t k = 0; k < splits; ++k) s += __ldg(ws + k * stride + i);
    out[i] = accumulate_into ? out[i] + s : s;
  }
}

__global__ void fill_kernel(float* __restrict__ out, int64_t count, float v) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out[i] = v;
}

// ---------------------------------------------------------------------------------------------
// Work split (pure function of the sizes)
// ---------------------------------------------------------------------------------------------

enum class Path { kMma, kDiagBf16, kGeneric };

Path choose_path(lhcal_mode mode, lhcal_dtype dtype, int32_t groups) {
  if (dtype == LHCAL_BF16 && mode != LHCAL_DIAG) return Path::kMma;
  if (dtype == LHCAL_BF16 && mode == LHCAL_DIAG && groups == 1) return Path::kDiagBf16;
  return Path::kGeneric;
}

struct Split {
  int64_t splits;   // CTAs along tokens
  int64_t per;      // tokens per split
};

// Token ranges so that splits * ctas_per_split does not exceed target_ctas (one wave of the
// resident CTAs; a second, nearly empty wave would double the time).
Split token_split(int64_t tokens, int64_t ctas_per_split, int64_t target_ctas, int64_t granule) {
  Split s;
  if (tokens <= 0) return {1, granule};
  int64_t want = imax64(1, target_ctas / imax64(ctas_per_split, 1));
  want = min(want, ceil_div(tokens, granule));
  s.per = ceil_div(ceil_div(tokens, want), granule) * granule;
  s.splits = ceil_div(tokens, s.per);
  return s;
}

// resident: CTAs per SM of the tensor-core variant launched (MmaCfg::kResident).
Split split_for(Path path, lhcal_mode mode, int64_t tokens, int64_t cin, int resident = 3) {
  switch (path) {
    case Path::kMma:
      return token_split(tokens, ceil_div(cin, kSlabCols), resident * kNumSms, kTileTok);
    case Path::kDiagBf16:
      return token_split(tokens, ceil_div(cin, kDiagCols), 8 * kNumSms, kDiagUnroll);
    default:
      return token_split(tokens, cin / kBlock, 4 * kNumSms, kGenTok);
  }
}

// Dense bf16 FULL / ACT: when the slabs alone nearly fill a wave, clusters of cs CTAs (cs <= 8)
// split each slab's tokens and reduce in distributed shared memory (no workspace, one launch);
// otherwise token splits write partials that reduce_partials_kernel sums.
struct DensePlan {
  bool cluster;
  int cs;
  int64_t splits;
  int64_t per;
};

DensePlan dense_plan(lhcal_mode mode, int64_t tokens, int64_t cin, int resident, double cluster_fill) {
  const int64_t slabs = ceil_div(cin, kSlabCols);
  const int64_t slots = static_cast<int64_t>(resident) * kNumSms;
  if (tokens > 0 && static_cast<double>(imin64(slabs * 8, slots)) >= cluster_fill * static_cast<double>(slots)) {
    int cs = 8;
    while (cs > 1 && slabs * cs > slots) cs /= 2;
    const int64_t per = ceil_div(ceil_div(tokens, cs), kTileTok) * kTileTok;
    return {true, cs, cs, per};
  }
  const Split sp = split_for(Path::kMma, mode, tokens, cin, resident);
  return {false, 0, sp.splits, sp.per};
}

size_t floats_per_split(lhcal_mode mode, int64_t cin) {
  const int64_t nblk = cin / kBlock;
  if (mode == LHCAL_DIAG) return static_cast<size_t>(cin);
  return static_cast<size_t>(nblk * 256 * (mode == LHCAL_ACT_AWARE ? 2 : 1));
}

lhcal_status launch_fill(float* out, int64_t count, float v, cudaStream_t stream) {
  if (count <= 0) return LHCAL_OK;
  const int64_t blocks = imin64(ceil_div(count, 256), 4 * kNumSms);
  fill_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(out, count, v);
  return check_launch("fill");
}

lhcal_status launch_reduce(const float* ws, int64_t splits, int64_t stride, int64_t count, float* out,
                           int accumulate_into, cudaStream_t stream) {
  const int64_t blocks = imin64(ceil_div(count, 256), 8 * kNumSms);
  reduce_partials_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(ws, splits, stride, count, out,
                                                                             accumulate_into);
  return check_launch("reduce partials");
}

template <bool ACT, bool QUANT>
lhcal_status launch_mma(const void* x, const void* xq, int64_t tokens, int64_t cin, int64_t ldx,
                        int32_t groups, const int32_t* offs, const int32_t* ids, int accumulate_into,
                        float* h, float* p, float* ws, cudaStream_t stream, const float* act_gx) {
  using Cfg = MmaCfg<ACT, QUANT>;
  // Allow up to the per-CTA maximum (the launch size decides occupancy). Set on every call with
  // the same value: cheap, thread-safe, and correct whichever device is current.
  constexpr int kMaxDynSmem = 227 * 1024;
  for (const void* fn : {reinterpret_cast<const void*>(accum_mma_kernel<ACT, QUANT, false>),
                         reinterpret_cast<const void*>(accum_mma_kernel<ACT, QUANT, true>)}) {
    const cudaError_t attr = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
    if (attr != cudaSuccess) return fail(LHCAL_ERR_CUDA, "accumulate: %s", cudaGetErrorString(attr));
  }
  const int64_t slabs = ceil_div(cin, kSlabCols);
  const int64_t nblk = cin / kBlock;
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  const auto* xqb = static_cast<const __nv_bfloat16*>(Cfg::kTwo ? xq : x);
  if (offs != nullptr) {
    // One persistent wave of resident CTAs dealt the (slab, expert) pairs round-robin; more CTAs
    // (several waves) only when a CTA's item ranges would not fit its shared-memory staging.
    const int64_t total = static_cast<int64_t>(groups) * slabs;
    const int64_t ctas = imin64(total, imax64(static_cast<int64_t>(Cfg::kResident) * kNumSms,
                                              ceil_div(total, kMaxStagedItems)));
    const size_t smem = Cfg::kSmem + static_cast<size_t>(ceil_div(total, ctas)) * sizeof(int4);
    accum_mma_kernel<ACT, QUANT, false><<<static_cast<unsigned>(ctas), kMmaThreads, smem, stream>>>(
        xb, xqb, tokens, cin, ldx, offs, ids, 0, total, groups, h, p, nblk * 256, accumulate_into, act_gx);
    return check_launch("accumulate (grouped, tensor cores)");
  }
  const DensePlan pl = dense_plan(ACT ? LHCAL_ACT_AWARE : LHCAL_FULL, tokens, cin, Cfg::kResident, Cfg::kClusterFill);
  if (pl.cluster) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(slabs), static_cast<unsigned>(pl.cs));
    cfg.blockDim = dim3(kMmaThreads);
    cfg.dynamicSmemBytes = Cfg::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 1;
    at[0].val.clusterDim.y = static_cast<unsigned>(pl.cs);
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, accum_mma_kernel<ACT, QUANT, true>, xb, xqb, tokens, cin, ldx,
                                             static_cast<const int32_t*>(nullptr), static_cast<const int32_t*>(nullptr),
                                             pl.per, static_cast<int64_t>(1), static_cast<int64_t>(0), h, ACT ? p : h,
                                             static_cast<int64_t>(0), accumulate_into, act_gx);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(LHCAL_ERR_CUDA, "accumulate (tensor cores, clusters): %s", cudaGetErrorString(e));
    }
    return check_launch("accumulate (tensor cores, clusters)");
  }
  const int64_t per_split = nblk * 256;
  float* ws_h = ws;
  float* ws_p = ws + pl.splits * per_split;
  const dim3 grid(static_cast<unsigned>(slabs), static_cast<unsigned>(pl.splits));
  accum_mma_kernel<ACT, QUANT, false><<<grid, kMmaThreads, Cfg::kSmem, stream>>>(
      xb, xqb, tokens, cin, ldx, nullptr, nullptr, pl.per, 1, 0, ws_h, ws_p, per_split, 0, act_gx);
  lhcal_status st = check_launch("accumulate (tensor cores)");
  if (st != LHCAL_OK) return st;
  st = launch_reduce(ws_h, pl.splits, per_split, per_split, h, accumulate_into, stream);
  if (st != LHCAL_OK || !ACT) return st;
  return launch_reduce(ws_p, pl.splits, per_split, per_split, p, accumulate_into, stream);
}

template <typename T, int MODE>
lhcal_status launch_generic(const void* x, const void* xq, int64_t tokens, int64_t cin, int64_t ldx,
                            int32_t groups, const int32_t* offs, const int32_t* ids, int accumulate_into,
                            float* h, float* p, float* ws, cudaStream_t stream) {
  const int64_t nblk = cin / kBlock;
  const int64_t per_group = (MODE == LHCAL_DIAG) ? cin : nblk * 256;
  const auto* xt = static_cast<const T*>(x);
  const auto* xqt = static_cast<const T*>(MODE == LHCAL_ACT_AWARE ? xq : x);
  if (offs != nullptr) {
    const dim3 grid(static_cast<unsigned>(nblk), static_cast<unsigned>(groups));
    accum_generic_kernel<T, MODE><<<grid, 256, 0, stream>>>(xt, xqt, tokens, cin, ldx, offs, ids, 0, h, p,
                                                            per_group, accumulate_into);
    return check_launch("accumulate (grouped)");
  }
  const Split sp = split_for(Path::kGeneric, MODE == LHCAL_ACT_AWARE ? LHCAL_ACT_AWARE : LHCAL_FULL, tokens, cin);
  float* ws_h = ws;
  float* ws_p = ws + sp.splits * per_group;
  const dim3 grid(static_cast<unsigned>(nblk), static_cast<unsigned>(sp.splits));
  accum_generic_kernel<T, MODE><<<grid, 256, 0, stream>>>(xt, xqt, tokens, cin, ldx, nullptr, nullptr, sp.per,
                                                          ws_h, ws_p, per_group, 0);
  lhcal_status st = check_launch("accumulate");
  if (st != LHCAL_OK) return st;
  st = launch_reduce(ws_h, sp.splits, per_group, per_group, h, accumulate_into, stream);
  if (st != LHCAL_OK || MODE != LHCAL_ACT_AWARE) return st;
  return launch_reduce(ws_p, sp.splits, per_group, per_group, p, accumulate_into, stream);
}

}  // namespace

size_t accumulate_workspace_bytes(lhcal_mode mode, lhcal_dtype dtype, int64_t tokens, int64_t cin,
                                  int32_t groups, bool quant) {
  if (groups != 1 || tokens <= 0) return 0;
  const Path path = choose_path(mode, dtype, groups);
  if (path == Path::kMma) {
    DensePlan pl;
    if (mode == LHCAL_ACT_AWARE && quant)
      pl = dense_plan(mode, tokens, cin, MmaCfg<true, true>::kResident, MmaCfg<true, true>::kClusterFill);
    else if (mode == LHCAL_ACT_AWARE)
      pl = dense_plan(mode, tokens, cin, MmaCfg<true, false>::kResident, MmaCfg<true, false>::kClusterFill);
    else
      pl = dense_plan(mode, tokens, cin, MmaCfg<false, false>::kResident, MmaCfg<false, false>::kClusterFill);
    return pl.cluster ? 0 : static_cast<size_t>(pl.splits) * floats_per_split(mode, cin) * sizeof(float);
  }
  const Split sp = split_for(path, mode, tokens, cin);
  return static_cast<size_t>(sp.splits) * floats_per_split(mode, cin) * sizeof(float);
}

lhcal_status launch_accumulate(lhcal_mode mode, lhcal_dtype dtype, const void* x, const void* xq,
                               int64_t tokens, int64_t cin, int64_t ldx, int32_t groups,
                               const int32_t* group_offsets, const int32_t* token_ids, int32_t flags,
                               float* h, float* p, void* workspace, cudaStream_t stream, const float* act_gx) {
  const int acc_into = (flags & LHCAL_ACCUM_OVERWRITE) ? 0 : 1;
  const int64_t nblk = cin / kBlock;
  const int64_t out_count = static_cast<int64_t>(groups) * (mode == LHCAL_DIAG ? cin : nblk * 256);
  if (group_offsets == nullptr && tokens == 0) {
    if (acc_into) return LHCAL_OK;
    lhcal_status st = launch_fill(h, out_count, 0.f, stream);
    if (st != LHCAL_OK || mode != LHCAL_ACT_AWARE) return st;
    return launch_fill(p, out_count, 0.f, stream);
  }
  float* ws = static_cast<float*>(workspace);
  const Path path = choose_path(mode, dtype, groups);
  if (act_gx != nullptr && path != Path::kMma)
    return fail(LHCAL_ERR_UNSUPPORTED, "the fused input quantizer needs bf16 activations");
  if (path == Path::kMma) {
    if (mode == LHCAL_ACT_AWARE && act_gx != nullptr)
      return launch_mma<true, true>(x, nullptr, tokens, cin, ldx, groups, group_offsets, token_ids, acc_into, h, p,
                                    ws, stream, act_gx);
    if (mode == LHCAL_ACT_AWARE)
      return launch_mma<true, false>(x, xq, tokens, cin, ldx, groups, group_offsets, token_ids, acc_into, h, p, ws,
                                     stream, nullptr);
    return launch_mma<false, false>(x, xq, tokens, cin, ldx, groups, group_offsets, token_ids, acc_into, h, p, ws,
                                    stream, nullptr);
  }
  if (path == Path::kDiagBf16) {
    const Split sp = split_for(path, mode, tokens, cin);
    const dim3 grid(static_cast<unsigned>(ceil_div(cin, kDiagCols)), static_cast<unsigned>(sp.splits));
    accum_diag_kernel<<<grid, kDiagThreads, 0, stream>>>(static_cast<const __nv_bfloat16*>(x), tokens, cin, ldx,
                                                         sp.per, ws);
    lhcal_status st = check_launch("accumulate (diagonal)");
    if (st != LHCAL_OK) return st;
    return launch_reduce(ws, sp.splits, cin, cin, h, acc_into, stream);
  }
#define LHCAL_GEN(T, M) \
  return launch_generic<T, M>(x, xq, tokens, cin, ldx, groups, group_offsets, token_ids, acc_into, h, p, ws, stream)
  if (dtype == LHCAL_F32) {
    if (mode == LHCAL_FULL) LHCAL_GEN(float, LHCAL_FULL);
    if (mode == LHCAL_ACT_AWARE) LHCAL_GEN(float, LHCAL_ACT_AWARE);
    LHCAL_GEN(float, LHCAL_DIAG);
  }
  LHCAL_GEN(__nv_bfloat16, LHCAL_DIAG);
#undef LHCAL_GEN
}

}  // namespace lhcal
