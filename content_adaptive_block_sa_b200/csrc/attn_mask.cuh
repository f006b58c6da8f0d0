// Element mask and list addressing shared by the attention kernels.
// Internal header.
#pragma once

#include "sa_common.cuh"

namespace sa {

constexpr int kMaxHeads = 256;

// Everything an attention kernel needs to know about the mask.
struct MaskArgs {
  int kind;                 // SA_MASK_GZIP / SA_MASK_GIST
  int T;                    // query/key tiles
  const int32_t* trp;       // tile CSR row pointers  [lists*(T+1)]
  const int32_t* tcol;      // key tiles
  const int8_t* tkind;      // kinds
  const int32_t* tcp;       // tile CSC pointers      [lists*(T+1)]
  const int32_t* trow;      // query tiles
  const int8_t* tkind_t;
  // gzip
  const uint32_t* bits;     // [batch*3*B*words]
  int B, b, words;
  int wb;                   // window w in blocks
  // gzip, b = 64, tensor-core forward ("pair mode"): a 128-row query tile
  // holds two 64-row query blocks and a 128-key tile two 64-key blocks.
  // Per list l: P pairs of query blocks pair_q[l * P + k] = qa | qb << 16
  // (qb = 0xffff: none); the visits of pair k are visits[pair_ptr[l * (P + 1)
  // + k] .. pair_ptr[l * (P + 1) + k + 1]) (absolute), each j1 | j2 << 12 |
  // vis << 24 with j2 = 0xfff for none and vis bits (qa sees j1, qb sees j1,
  // qa sees j2, qb sees j2).
  int pair, P;
  const int32_t* pair_q;
  const int32_t* pair_ptr;
  const int32_t* visits;
  // gist
  const int32_t* perm;      // physical -> logical
  const uint32_t* gist_bits;
  const int32_t* far_idx;   // sinks + gists in logical order (physical indices)
  const int32_t* far_ptr;   // [T+1] far keys below each key tile
  int sinks, window;
  uint8_t head_class[kMaxHeads];  // gzip: class of each query head
};

// Pointers, shapes and strides (elements) of one attention call.
struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  const void* dout;
  float* dq;
  float* dk;
  float* dv;
  float* delta;  // [Bt, Hq, N] rowsum(dO * O)
  int Bt, N, Hq, Hkv;
  float scale;
  int64_t qs[3], ks[3], vs[3], os[3];
  DeviceStatus* status;
};

// Index of the list used by (batch row, query head).
__device__ __forceinline__ int list_of(const MaskArgs& m, int bt, int h) {
  return m.kind == SA_MASK_GZIP ? bt * 3 + m.head_class[h] : 0;
}

// Is physical key q visible from physical query p (both < N)?
__device__ __forceinline__ bool element_visible(const MaskArgs& m, int list, int p, int q) {
  if (m.kind == SA_MASK_GZIP) {
    if (q > p) return false;
    const uint32_t* row = m.bits + ((int64_t)list * m.B + p / m.b) * m.words;
    const int j = q / m.b;
    return (row[j >> 5] >> (j & 31)) & 1u;
  }
  const int i = m.perm[p], j = m.perm[q];
  if (j > i) return false;
  const bool g = (m.gist_bits[j >> 5] >> (j & 31)) & 1u;
  return j < m.sinks || g || (i - j) < m.window;
}

}  // namespace sa
