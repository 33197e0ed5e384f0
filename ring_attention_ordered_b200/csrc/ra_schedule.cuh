// Work units of the forward kernels and their order, shared by the bf16 and
// FP8 forward kernels (which take them from a launch-wide queue in this
// order, ra_fwd_roles.cuh).  The parameter structs of both carry
// the same scheduling fields (B, Hq, Hkv, group, n_ring, blk_len, causal,
// tiles_per_blk, pair_heads, head_slots, pairs_per_blk, head_major,
// total_units), so these helpers are templates over the struct.
//
// The ring order follows "Ring Attention 环注意力" (L3 definition, L4 §4.2):
// the query block of host i visits K/V blocks (i - t) mod n_ring; under
// causal masking later blocks are skipped (L4 §4.5, limitation 2), and units
// are ordered longest first for load balance (L4 §4.5, limitation 3).
#pragma once

namespace ra {

struct Unit {
  int b, kvh, blk;
  int h[2];
  int qt[2];       // tile index inside ring block blk
  int valid1;
  int qt_last;
  int n_kv;        // K/V tiles visited, in ring order
};

// Unit order.  head_major = 0: all units sorted longest first across every
// (batch, head).  head_major = 1: (batch, K/V head) major, longest first
// inside each K/V head, so the CTAs running at any moment share one or two
// K/V heads whose tiles stay in L2 instead of streaming from HBM.
template <class P>
__device__ __forceinline__ Unit decode_unit(const P& p, int u) {
  Unit x;
  const int tpb = p.tiles_per_blk;
  if (p.pair_heads) {
    const int n_tiles = p.n_ring * tpb;
    int r, rem;
    if (p.head_major) {
      const int per_head = n_tiles * p.head_slots;
      rem = u / per_head;                       // b * Hkv + kvh
      const int v = u % per_head;
      r = v / p.head_slots;
      rem = rem * p.head_slots + v % p.head_slots;
    } else {
      const int per_tile = p.B * p.Hkv * p.head_slots;
      r = u / per_tile;
      rem = u % per_tile;
    }
    const int gt = n_tiles - 1 - r;   // longest first
    x.blk = gt / tpb;
    const int local = gt % tpb;
    const int slot = rem % p.head_slots;
    rem /= p.head_slots;
    x.kvh = rem % p.Hkv;
    x.b = rem / p.Hkv;
    x.h[0] = x.kvh * p.group + 2 * slot;
    x.h[1] = x.h[0] + 1;
    x.valid1 = (2 * slot + 1) < p.group;
    x.qt[0] = x.qt[1] = local;
  } else {
    int r, bh;
    if (p.head_major) {
      const int per_head = p.n_ring * p.pairs_per_blk;
      bh = u / per_head;
      r = u % per_head;
    } else {
      const int per_pair = p.B * p.Hq;
      r = u / per_pair;
      bh = u % per_pair;
    }
    x.b = bh / p.Hq;
    x.h[0] = x.h[1] = bh % p.Hq;
    x.kvh = x.h[0] / p.group;
    const int ppb = p.pairs_per_blk;
    x.blk = p.n_ring - 1 - r / ppb;
    const int pr = ppb - 1 - r % ppb;
    x.qt[0] = 2 * pr;
    x.qt[1] = 2 * pr + 1;
    x.valid1 = x.qt[1] < tpb;
  }
  x.qt_last = x.valid1 ? max(x.qt[0], x.qt[1]) : x.qt[0];
  x.n_kv = p.causal ? (x.blk * tpb + x.qt_last + 1) : (p.n_ring * tpb);
  return x;
}

// K/V tiles of a unit in visit order.  The unit's own block comes first
// (ring step t = 0), then blocks (i - t) mod n_ring for t = 1, 2, ...; inside
// a block the tiles run in ascending order, and under causal masking the own
// block stops at the unit's last query tile while later blocks are skipped.
struct KvIter {
  int jb;      // ring block of the current tile
  int kl;      // tile index inside that block
  int end;     // tiles of this block to visit
  template <class P>
  __device__ __forceinline__ void start(const P& p, const Unit& x) {
    jb = x.blk;
    kl = 0;
    end = p.causal ? (x.qt_last + 1) : p.tiles_per_blk;
  }
  template <class P>
  __device__ __forceinline__ void next(const P& p) {
    if (++kl == end) {
      kl = 0;
      jb = (jb == 0) ? p.n_ring - 1 : jb - 1;
      end = p.tiles_per_blk;
    }
  }
};

}  // namespace ra
