// Bounds-checked debug build of the tensor-core kernels.
//
// Compiled with -DMLSTM_BOUNDS_CHECK (the library libmlstm_checked.so), the mLSTM prefill's gate
// preparation, segment-summary and walk kernels and the GDN-2 chunk kernels check, before making
// it, every plain global access against the extent of its buffer, every TMA copy's coordinates
// against the copy rules (the innermost coordinate on a 16-byte boundary, a store from
// non-negative coordinates, a box that overlaps its tensor) and every staging-tile offset of the
// h store against the tile.  A failing check skips the access, sets bit 2 (value 4) of the
// workspace error word and records the first failure (site, index, extent) at bytes 16..39 of
// the workspace (the GDN-2 kernels: of their own workspace's header); the call's status is then
// MLSTM_ERR_BOUNDS.  Nothing traps.  In the normal build every check is the constant true and
// compiles away.
#pragma once

namespace mlstm {

// Where a check sits (recorded with a failure).
enum BoundsSite : int {
  BS_NONE = 0,
  BS_GATE_INPUT = 1,     // ig / fg read by the gate preparation
  BS_GATE_PLANES = 2,    // gb / gx / gxc rows written by the gate preparation
  BS_GATE_CHUNK = 3,     // cg / cxm entries written by the gate preparation
  BS_SEG_TMA = 4,        // K, V loads of the segment summaries
  BS_SEG_CHUNK = 5,      // cg / cxm read by the segment summaries
  BS_SEG_SCALARS = 6,    // segA / segB written
  BS_SEG_DC = 7,         // summary rows dC written
  BS_SEG_DN = 8,         // summary n (dn) written
  BS_WALK_START = 9,     // C0 / n0 / m0, segA / segB, dn read for the start state
  BS_WALK_SUM_TMA = 10,  // summary tiles loaded into the stage area
  BS_WALK_TMA = 11,      // Q, K, V loads of the walk
  BS_WALK_GATES = 12,    // gate planes and chunk entries read by the walk's producer
  BS_WALK_OGATE = 13,    // output-gate rows read
  BS_WALK_H_STAGE = 14,  // staging tile of h (shared memory)
  BS_WALK_H_TMA = 15,    // h tile stores
  BS_WALK_FINAL = 16,    // C_out / n_out / m_out written
  BS_WALK_BIAS = 17,     // scalar-normaliser bias read
  BS_GDN_INPUT = 18,     // GDN-2 chunk prep: q, k, g, b, v, w rows read
  BS_GDN_SLOT = 19,      // GDN-2 chunk prep: writes into the chunk's workspace slot
  BS_GDN_COPY = 20,      // GDN-2 chunk scan: slot copied into a stage
  BS_GDN_STATE = 21,     // GDN-2 chunk scan: S0 read, S_out written
  BS_GDN_OUT = 22,       // GDN-2 chunk scan: o written
};

struct BoundsRecord {
  int site, count;
  long long index, extent;
};

#ifdef MLSTM_BOUNDS_CHECK
constexpr bool kBoundsChecked = true;
static __device__ __noinline__ bool bounds_fail(unsigned int* err, int site, long long index, long long extent) {
  BoundsRecord* r = reinterpret_cast<BoundsRecord*>(reinterpret_cast<char*>(err) + 16);
  atomicOr(err, 4u);
  if (atomicAdd(&r->count, 1) == 0) {
    r->site = site;
    r->index = index;
    r->extent = extent;
  }
  return false;
}
// 0 <= index < extent
__device__ __forceinline__ bool in_bounds(unsigned int* err, int site, long long index, long long extent) {
  return (unsigned long long)index < (unsigned long long)extent || bounds_fail(err, site, index, extent);
}
// a condition, with the value and limit recorded when it fails
__device__ __forceinline__ bool bounds_require(unsigned int* err, int site, bool ok, long long index,
                                               long long extent) {
  return ok || bounds_fail(err, site, index, extent);
}
// a TMA box at (x, y) of a tensor with dims (d0, d1) and box rows `rows`: x on a 16-byte
// boundary (`align` elements) and inside d0; stores start at y >= 0, loads may start up to
// `rows` - 1 rows above the tensor (zero fill) but must overlap it
__device__ __forceinline__ bool tma_box_ok(unsigned int* err, int site, int x, int y, int align, long long d0,
                                           long long d1, int rows, bool store) {
  if (x % align != 0 || x < 0 || x >= d0) return bounds_fail(err, site, x, d0);
  if (store ? (y < 0 || y >= d1) : (y <= -rows || y >= d1)) return bounds_fail(err, site, y, d1);
  return true;
}
#else
constexpr bool kBoundsChecked = false;
__device__ __forceinline__ bool in_bounds(unsigned int*, int, long long, long long) { return true; }
__device__ __forceinline__ bool bounds_require(unsigned int*, int, bool, long long, long long) { return true; }
__device__ __forceinline__ bool tma_box_ok(unsigned int*, int, int, int, int, long long, long long, int, bool) {
  return true;
}
#endif

}  // namespace mlstm
