// Gist-scored selective unfolding at decode.
//
// "Simplified Sparse Attention via Gist Tokens" (abstract): the current query
// is scored against the small set of gist keys only, the top-k chunks are
// unfolded by bringing back their raw tokens, and attention runs over them;
// "Forget, Then Recall: ... Gist Sparse Attention" (abstract): compress into
// gists, select the most relevant gists, restore the corresponding raw chunks.
//
// Per (sequence, KV head g) with query heads h in the group:
//   1. gist pass (split over gist slices): s_h,c = q_h . gk_c * scale for
//      every gist c; the selection score sum_h s_h,c goes to the workspace and
//      the same logits feed the gist part of the attention as a partial
//      (max m, sum l, unnormalised o) per head and slice. Gist K and V are
//      streamed once.
//   2. select: top_k eligible chunks (wholly before the window) by score,
//      ties to the lower index, written ascending (-1 padded). The score is
//      the sum of the group's logits, or (sum-of-probabilities rule) the sum
//      of each head's softmax over all gists, from per-head logits the gist
//      pass stores and the heads' gist-slice partials; the top-p rule keeps
//      the shortest score-ordered prefix whose softmax over the eligible
//      chunks reaches p.
//   3. raw pass (split over the unfolded keys): the same partials over the
//      raw tokens of the selected chunks followed by the last `window`
//      tokens.
//   4. combine the partials of every slice into O (bf16) and LSE (fp32).
// Keys and values are read with 16-byte loads, 16 lanes per 256-byte row.
#include <cuda.h>

#include <mutex>

#include "sa_common.cuh"

namespace sa {

constexpr int kDecD = 128;
constexpr int kDecMaxRep = 8;   // query heads per KV head
constexpr int kGistSlice = 256;
constexpr int kRawSlice = 256;
constexpr int kDecThreads = 128;

struct DecodeArgs {
  const __nv_bfloat16 *q, *gk, *gv, *kc, *vc;
  int32_t* sel;
  __nv_bfloat16* o;
  float* lse;
  float* scores;   // [n_seq, Hkv, G]
  float* part;     // [n_seq, Hq, n_part, 2 + D]
  float* logits;   // [n_seq, Hq, G] scaled logits (sum-of-probabilities rule)
  int rule;
  float top_p;
  // gist of gists: level-2 gists, their selection, and (selecting level 1)
  // the kept groups whose level-1 gists are the candidates
  const __nv_bfloat16 *g2k, *g2v;
  int64_t g2s[3];
  int32_t* sel2;
  const int32_t* cand_groups;
  int n2, fanout, top_k2;
  int n_seq, cache_len, chunk, G, top_k, window, Hq, Hkv, rep;
  int n_gslices, n_rslices, n_part;
  float scale;
  int64_t qs[2], gs[3], cs[3], os[2];
};

__device__ __forceinline__ void bf16x8_to_float(const uint4& u, float* f) {
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(b[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// Online-softmax state of one half-warp for the group's heads; each lane
// holds 8 of the 128 output dimensions.
template <int REP>
struct HalfState {
  float m[REP], l[REP], o[REP][8];
  __device__ void init() {
#pragma unroll
    for (int h = 0; h < REP; ++h) {
      m[h] = -INFINITY;
      l[h] = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) o[h][i] = 0.f;
    }
  }
};

// Processes keys [e0, e1) of a key list given by `row` (returns k/v row
// pointers) and writes one partial per head to `out` (slot `slot`).
// heads_of(e) gives the query heads (bits) that see key e.
template <int REP, typename RowFn, typename HeadsFn>
__device__ void attend_slice(const DecodeArgs& a, const float (*qf)[kDecD], int e0, int e1,
                             RowFn row, HeadsFn heads_of, float* score_out, float* logit_out,
                             int seq, int g, int slot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int half = lane >> 4, hl = lane & 15;  // 16 lanes per key row
  HalfState<REP> st;
  st.init();
  float qreg[REP][8];
#pragma unroll
  for (int h = 0; h < REP; ++h)
#pragma unroll
    for (int i = 0; i < 8; ++i) qreg[h][i] = qf[h][hl * 8 + i];
  const int nw = blockDim.x >> 5;
  for (int base = e0 + warp * 2; base < e1; base += nw * 2) {
    const int e = base + half;
    const bool valid = e < e1;
    float kf[8], vf[8];
    if (valid) {
      const __nv_bfloat16 *kr, *vr;
      row(e, kr, vr);
      bf16x8_to_float(*reinterpret_cast<const uint4*>(kr + hl * 8), kf);
      bf16x8_to_float(*reinterpret_cast<const uint4*>(vr + hl * 8), vf);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) kf[i] = vf[i] = 0.f;
    }
    float s[REP];
    float ssum = 0.f;
#pragma unroll
    for (int h = 0; h < REP; ++h) {
      float t = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) t = fmaf(qreg[h][i], kf[i], t);
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
      s[h] = t * a.scale;
      ssum += s[h];
    }
    if (valid && score_out != nullptr && hl == 0) score_out[e] = ssum;
    if (valid && logit_out != nullptr && hl == 0)
#pragma unroll
      for (int h = 0; h < REP; ++h) logit_out[(int64_t)h * a.G + e] = s[h];
    if (!valid) continue;
    const uint32_t hv = heads_of(e);
#pragma unroll
    for (int h = 0; h < REP; ++h) {
      if (!((hv >> h) & 1u)) continue;
      const float mnew = fmaxf(st.m[h], s[h]);
      const float alpha = expf(st.m[h] - mnew);
      const float p = expf(s[h] - mnew);
      st.l[h] = st.l[h] * alpha + p;
#pragma unroll
      for (int i = 0; i < 8; ++i) st.o[h][i] = fmaf(p, vf[i], st.o[h][i] * alpha);
      st.m[h] = mnew;
    }
  }
  // combine the 2 * nwarps half-warp states through shared memory
  __shared__ float red_m[8][kDecMaxRep], red_l[8][kDecMaxRep];
  __shared__ float red_o[kDecMaxRep][kDecD];
  const int hw = warp * 2 + half;  // 0..7
  if (hl == 0)
#pragma unroll
    for (int h = 0; h < REP; ++h) { red_m[hw][h] = st.m[h]; red_l[hw][h] = st.l[h]; }
  for (int x = threadIdx.x; x < REP * kDecD; x += blockDim.x) red_o[x / kDecD][x % kDecD] = 0.f;
  __syncthreads();
  float M[REP], scale_me[REP];
#pragma unroll
  for (int h = 0; h < REP; ++h) {
    M[h] = -INFINITY;
    for (int t = 0; t < 2 * nw; ++t) M[h] = fmaxf(M[h], red_m[t][h]);
    scale_me[h] = (st.m[h] == -INFINITY) ? 0.f : expf(st.m[h] - M[h]);
  }
#pragma unroll
  for (int h = 0; h < REP; ++h)
#pragma unroll
    for (int i = 0; i < 8; ++i) atomicAdd(&red_o[h][hl * 8 + i], st.o[h][i] * scale_me[h]);
  __syncthreads();
  for (int x = threadIdx.x; x < REP * kDecD; x += blockDim.x) {
    const int h = x / kDecD, c = x % kDecD;
    float* dst = a.part + (((int64_t)seq * a.Hq + g * a.rep + h) * a.n_part + slot) * (2 + kDecD);
    dst[2 + c] = red_o[h][c];
    if (c == 0) {
      float L = 0.f;
      for (int t = 0; t < 2 * nw; ++t)
        if (red_m[t][h] != -INFINITY) L += red_l[t][h] * expf(red_m[t][h] - M[h]);
      dst[0] = M[h];
      dst[1] = L;
    }
  }
}

__device__ void load_group_q(const DecodeArgs& a, int seq, int g, float (*qf)[kDecD]) {
  for (int x = threadIdx.x; x < a.rep * kDecD; x += blockDim.x) {
    const int h = x / kDecD, c = x % kDecD;
    qf[h][c] = __bfloat162float(a.q[seq * a.qs[0] + (int64_t)(g * a.rep + h) * a.qs[1] + c]);
  }
  __syncthreads();
}

template <int REP>
__global__ void __launch_bounds__(kDecThreads) decode_gist_kernel(DecodeArgs a) {
  __shared__ float qf[kDecMaxRep][kDecD];
  const int slice = blockIdx.x, g = blockIdx.y, seq = blockIdx.z;
  load_group_q(a, seq, g, qf);
  const __nv_bfloat16* gk = a.gk + seq * a.gs[0] + (int64_t)g * a.gs[1];
  const __nv_bfloat16* gv = a.gv + seq * a.gs[0] + (int64_t)g * a.gs[1];
  const int64_t rs = a.gs[2];
  auto row = [&](int e, const __nv_bfloat16*& kr, const __nv_bfloat16*& vr) {
    kr = gk + e * rs;
    vr = gv + e * rs;
  };
  const int e0 = slice * kGistSlice, e1 = min(a.G, e0 + kGistSlice);
  float* sc = a.scores + ((int64_t)seq * a.Hkv + g) * a.G;
  float* lg = (a.rule == SA_SELECT_SUM_PROBS_PER_GROUP || a.rule == SA_SELECT_TOP_K_PER_HEAD)
                  ? a.logits + ((int64_t)seq * a.Hq + g * a.rep) * a.G
                  : nullptr;
  attend_slice<REP>(a, qf, e0, e1, row, [](int) { return 0xFFFFFFFFu; }, sc, lg, seq, g, slice);
}

// Order-preserving map of a float to an unsigned key, and back.
__device__ __forceinline__ uint32_t float_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

__global__ void __launch_bounds__(1024) decode_select_kernel(DecodeArgs a, int pow2) {
  extern __shared__ unsigned long long keys[];
  __shared__ int chosen[256];
  const int g = blockIdx.x, seq = blockIdx.y;
  __shared__ float lse_h[kDecMaxRep];
  __shared__ float red[32];
  __shared__ int n_keep_s;
  // per-head rule: blockIdx.x is the query head and its logits are the scores
  const bool per_head = a.rule == SA_SELECT_TOP_K_PER_HEAD;
  const float* sc = per_head ? a.logits + ((int64_t)seq * a.Hq + g) * a.G
                             : a.scores + ((int64_t)seq * a.Hkv + g) * a.G;
  const bool probs = a.rule == SA_SELECT_SUM_PROBS_PER_GROUP;
  const float* lg = a.logits + ((int64_t)seq * a.Hq + g * a.rep) * a.G;
  if (probs && threadIdx.x < a.rep) {
    // head h's log-sum-exp over all gists, from its gist-slice partials
    const float* p = a.part + ((int64_t)seq * a.Hq + g * a.rep + threadIdx.x) * a.n_part * (2 + kDecD);
    float M = -INFINITY;
    for (int t = 0; t < a.n_gslices; ++t) M = fmaxf(M, p[t * (2 + kDecD)]);
    float L = 0.f;
    for (int t = 0; t < a.n_gslices; ++t)
      if (p[t * (2 + kDecD)] != -INFINITY) L += p[t * (2 + kDecD) + 1] * expf(p[t * (2 + kDecD)] - M);
    lse_h[threadIdx.x] = M + logf(L);
  }
  __syncthreads();
  const int last_ok = a.cache_len - a.window;  // chunk c eligible iff (c+1)*chunk <= last_ok
  // level-1 selection of the gist of gists: candidate i is level-1 gist
  // i % fanout of kept group cg[i / fanout] (every kept group is eligible)
  const int32_t* cg = a.cand_groups ? a.cand_groups + ((int64_t)seq * a.Hkv + g) * a.top_k2 : nullptr;
  for (int i = threadIdx.x; i < pow2; i += blockDim.x) {
    unsigned long long kk = 0ull;
    const bool elig = cg ? (i < a.G && cg[i / a.fanout] >= 0)
                         : (i < a.G && (int64_t)(i + 1) * a.chunk <= last_ok);
    if (elig) {
      float v = sc[i];
      if (probs) {
        v = 0.f;
        for (int h = 0; h < a.rep; ++h) v += expf(lg[(int64_t)h * a.G + i] - lse_h[h]);
      }
      kk = ((unsigned long long)float_key(v) << 32) | (0xFFFFFFFFu - (uint32_t)i);
    }
    keys[i] = kk;
  }
  __syncthreads();
  // bitonic sort, descending
  for (int size = 2; size <= pow2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < pow2; i += blockDim.x) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0;
          const unsigned long long x = keys[i], y = keys[j];
          if ((x < y) == desc) { keys[i] = y; keys[j] = x; }
        }
      }
      __syncthreads();
    }
  }
  const int k = a.top_k;
  if (threadIdx.x == 0) n_keep_s = k;
  if (a.rule == SA_SELECT_TOP_P_PER_GROUP && k > 0 && keys[0] != 0ull) {
    // softmax over the eligible chunks (keys[0] holds the best score), then the
    // shortest prefix of the sorted keys whose probability reaches p
    const float smax = key_float((uint32_t)(keys[0] >> 32));
    float z = 0.f;
    for (int i = threadIdx.x; i < pow2; i += blockDim.x)
      if (keys[i] != 0ull) z += expf(key_float((uint32_t)(keys[i] >> 32)) - smax);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = z;
    __syncthreads();
    if (threadIdx.x == 0) {
      float Z = 0.f;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) Z += red[w];
      const float thr = a.top_p * Z;
      float cum = 0.f;
      int n = 0;
      for (int t = 0; t < k && t < pow2 && keys[t] != 0ull; ++t) {
        if (n > 0 && cum >= thr) break;
        cum += expf(key_float((uint32_t)(keys[t] >> 32)) - smax);
        ++n;
      }
      n_keep_s = n;
    }
  }
  __syncthreads();
  const int n_keep = n_keep_s;
  for (int t = threadIdx.x; t < k; t += blockDim.x)
    chosen[t] = (t < n_keep && t < pow2 && keys[t] != 0ull)
                    ? (int)(0xFFFFFFFFu - (uint32_t)(keys[t] & 0xFFFFFFFFull))
                    : 0x7FFFFFFF;
  __syncthreads();
  int32_t* out = a.sel + ((int64_t)seq * (per_head ? a.Hq : a.Hkv) + g) * k;
  for (int t = threadIdx.x; t < k; t += blockDim.x) {
    const int v = chosen[t];
    int rank = 0;
    for (int u = 0; u < k; ++u) rank += chosen[u] < v || (chosen[u] == v && u < t);
    out[rank] = (v == 0x7FFFFFFF) ? -1 : cg ? cg[v / a.fanout] * a.fanout + v % a.fanout : v;
  }
}

template <int REP>
__global__ void __launch_bounds__(kDecThreads) decode_raw_kernel(DecodeArgs a) {
  __shared__ float qf[kDecMaxRep][kDecD];
  __shared__ int sel_s[kDecMaxRep * 256];
  __shared__ int n_sel_s;
  const int slice = blockIdx.x, g = blockIdx.y, seq = blockIdx.z;
  // per-head rule: the group's heads' selections one after another (every
  // head takes the same number of chunks); a key of head hh's chunks is seen
  // by that head only
  const bool per_head = a.rule == SA_SELECT_TOP_K_PER_HEAD;
  const int nh = per_head ? a.rep : 1;
  const int32_t* sel = a.sel + ((int64_t)seq * a.Hkv + g) * nh * a.top_k;
  for (int t = threadIdx.x; t < nh * a.top_k; t += blockDim.x) sel_s[t] = sel[t];
  __syncthreads();
  if (threadIdx.x == 0) {
    int n = 0;
    for (int t = 0; t < a.top_k; ++t) n += sel_s[t] >= 0;
    n_sel_s = n;
  }
  load_group_q(a, seq, g, qf);
  const int head_keys = n_sel_s * a.chunk;
  const int n_chunk_keys = nh * head_keys;
  const int total = n_chunk_keys + a.window;
  const __nv_bfloat16* kc = a.kc + seq * a.cs[0] + (int64_t)g * a.cs[1];
  const __nv_bfloat16* vc = a.vc + seq * a.cs[0] + (int64_t)g * a.cs[1];
  const int64_t rs = a.cs[2];
  const int chunk = a.chunk, wstart = a.cache_len - a.window;
  const int ktop = a.top_k;
  auto row = [&](int e, const __nv_bfloat16*& kr, const __nv_bfloat16*& vr) {
    int pos;
    if (e < n_chunk_keys) {
      const int hh = e / head_keys, x = e - hh * head_keys;
      pos = sel_s[hh * ktop + x / chunk] * chunk + x % chunk;
    } else {
      pos = wstart + (e - n_chunk_keys);
    }
    kr = kc + pos * rs;
    vr = vc + pos * rs;
  };
  auto heads_of = [&](int e) -> uint32_t {
    return (per_head && e < n_chunk_keys) ? 1u << (e / head_keys) : 0xFFFFFFFFu;
  };
  const int e0 = min(total, slice * kRawSlice), e1 = min(total, e0 + kRawSlice);
  attend_slice<REP>(a, qf, e0, e1, row, heads_of, nullptr, nullptr, seq, g, a.n_gslices + slice);
}

// Gist of gists, step 1: every level-2 gist, its summed logit into scores
// (the level-2 score row) and its partial into slot `slice`.
template <int REP>
__global__ void __launch_bounds__(kDecThreads) hier_gist2_kernel(DecodeArgs a, float* scores2) {
  __shared__ float qf[kDecMaxRep][kDecD];
  const int slice = blockIdx.x, g = blockIdx.y, seq = blockIdx.z;
  load_group_q(a, seq, g, qf);
  const __nv_bfloat16* gk = a.g2k + seq * a.g2s[0] + (int64_t)g * a.g2s[1];
  const __nv_bfloat16* gv = a.g2v + seq * a.g2s[0] + (int64_t)g * a.g2s[1];
  const int64_t rs = a.g2s[2];
  auto row = [&](int e, const __nv_bfloat16*& kr, const __nv_bfloat16*& vr) {
    kr = gk + e * rs;
    vr = gv + e * rs;
  };
  const int e0 = slice * kGistSlice, e1 = min(a.n2, e0 + kGistSlice);
  attend_slice<REP>(a, qf, e0, e1, row, [](int) { return 0xFFFFFFFFu; },
                    scores2 + ((int64_t)seq * a.Hkv + g) * a.n2, nullptr, seq, g, slice);
}

// Step 2: the level-1 gists of the kept groups (a prefix of sel2: it is
// ascending, -1 padded), candidate e = level-1 gist e % fanout of group
// sel2[e / fanout]; summed logits into scores1 [.., top_k2 * fanout] and
// partials into the slots after step 1's.
template <int REP>
__global__ void __launch_bounds__(kDecThreads) hier_gist1_kernel(DecodeArgs a, float* scores1,
                                                                 int slot0) {
  __shared__ float qf[kDecMaxRep][kDecD];
  __shared__ int grp[256];
  __shared__ int n_grp_s;
  const int slice = blockIdx.x, g = blockIdx.y, seq = blockIdx.z;
  const int32_t* sel2 = a.sel2 + ((int64_t)seq * a.Hkv + g) * a.top_k2;
  for (int t = threadIdx.x; t < a.top_k2; t += blockDim.x) grp[t] = sel2[t];
  __syncthreads();
  if (threadIdx.x == 0) {
    int n = 0;
    for (int t = 0; t < a.top_k2; ++t) n += grp[t] >= 0;
    n_grp_s = n;
  }
  load_group_q(a, seq, g, qf);
  const int n_cand = n_grp_s * a.fanout, fo = a.fanout;
  const __nv_bfloat16* gk = a.gk + seq * a.gs[0] + (int64_t)g * a.gs[1];
  const __nv_bfloat16* gv = a.gv + seq * a.gs[0] + (int64_t)g * a.gs[1];
  const int64_t rs = a.gs[2];
  auto row = [&](int e, const __nv_bfloat16*& kr, const __nv_bfloat16*& vr) {
    const int j = grp[e / fo] * fo + e % fo;
    kr = gk + j * rs;
    vr = gv + j * rs;
  };
  const int e0 = min(n_cand, slice * kGistSlice), e1 = min(n_cand, e0 + kGistSlice);
  attend_slice<REP>(a, qf, e0, e1, row, [](int) { return 0xFFFFFFFFu; },
                    scores1 + ((int64_t)seq * a.Hkv + g) * a.top_k2 * fo, nullptr, seq, g,
                    slot0 + slice);
}

__global__ void decode_combine_kernel(DecodeArgs a) {
  const int h = blockIdx.x, seq = blockIdx.y, c = threadIdx.x;  // 128 threads
  const float* p = a.part + ((int64_t)seq * a.Hq + h) * a.n_part * (2 + kDecD);
  float M = -INFINITY;
  for (int t = 0; t < a.n_part; ++t) M = fmaxf(M, p[t * (2 + kDecD)]);
  float L = 0.f, acc = 0.f;
  for (int t = 0; t < a.n_part; ++t) {
    const float* q = p + t * (2 + kDecD);
    if (q[0] == -INFINITY) continue;
    const float w = expf(q[0] - M);
    L += q[1] * w;
    acc += q[2 + c] * w;
  }
  a.o[seq * a.os[0] + (int64_t)h * a.os[1] + c] = __float2bfloat16_rn(acc / L);
  if (c == 0) a.lse[(int64_t)seq * a.Hq + h] = M + logf(L);
}

// ------------------------------------------------------------- host side
struct DecodePlan {
  int n_gslices, n_rslices, n_part, pow2;
  size_t scores_off, part_off, logits_off, bytes;
};

DecodePlan decode_plan(const sa_decode_desc& d) {
  DecodePlan p{};
  p.n_gslices = (d.n_gists + kGistSlice - 1) / kGistSlice;
  const int heads = d.select_rule == SA_SELECT_TOP_K_PER_HEAD ? d.num_q_heads / d.num_kv_heads : 1;
  const int max_raw = heads * d.top_k * d.chunk + d.window;
  p.n_rslices = max(1, (max_raw + kRawSlice - 1) / kRawSlice);
  p.n_part = p.n_gslices + p.n_rslices;
  p.pow2 = 1;
  while (p.pow2 < d.n_gists) p.pow2 <<= 1;
  p.scores_off = kStatusBytes;
  size_t sb = (size_t)d.n_seq * d.num_kv_heads * d.n_gists * sizeof(float);
  p.part_off = p.scores_off + ((sb + 255) / 256) * 256;
  size_t pb = (size_t)d.n_seq * d.num_q_heads * p.n_part * (2 + kDecD) * sizeof(float);
  p.logits_off = p.part_off + ((pb + 255) / 256) * 256;
  size_t lb = (d.select_rule == SA_SELECT_SUM_PROBS_PER_GROUP ||
               d.select_rule == SA_SELECT_TOP_K_PER_HEAD)
                  ? (size_t)d.n_seq * d.num_q_heads * d.n_gists * sizeof(float)
                  : 0;
  p.bytes = p.logits_off + lb;
  return p;
}

template <int REP>
static cudaError_t decode_launch_rep(const DecodeArgs& a, const DecodePlan& pl, cudaStream_t s) {
  decode_gist_kernel<REP><<<dim3(pl.n_gslices, a.Hkv, a.n_seq), kDecThreads, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)pl.pow2 * sizeof(unsigned long long);
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(decode_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int sel_rows = a.rule == SA_SELECT_TOP_K_PER_HEAD ? a.Hq : a.Hkv;
  decode_select_kernel<<<dim3(sel_rows, a.n_seq), 1024, smem, s>>>(a, pl.pow2);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_raw_kernel<REP><<<dim3(pl.n_rslices, a.Hkv, a.n_seq), kDecThreads, 0, s>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<<<dim3(a.Hq, a.n_seq), kDecD, 0, s>>>(a);
  return cudaGetLastError();
}

bool decode_tc_supported(const sa_decode_desc& d);
cudaError_t launch_decode_tc(const sa_decode_desc& d, const void* q, const void* gk,
                             const void* gv, const void* kc, const void* vc, int32_t* sel, void* o,
                             float* lse, void* ws, float* logits, cudaStream_t s);

// The tensor-core kernel (one CTA per sequence and KV head) takes the shapes it
// supports; the four-pass CUDA-core kernels below take the rest.
cudaError_t launch_decode(const sa_decode_desc& d, const void* q, const void* gk, const void* gv,
                          const void* kc, const void* vc, int32_t* sel, void* o, float* lse,
                          void* ws, cudaStream_t s) {
  const DecodePlan pl = decode_plan(d);
  float* logits = (float*)((char*)ws + pl.logits_off);
  if (decode_tc_supported(d))
    return launch_decode_tc(d, q, gk, gv, kc, vc, sel, o, lse, ws, logits, s);
  DecodeArgs a{};
  a.q = (const __nv_bfloat16*)q;
  a.gk = (const __nv_bfloat16*)gk;
  a.gv = (const __nv_bfloat16*)gv;
  a.kc = (const __nv_bfloat16*)kc;
  a.vc = (const __nv_bfloat16*)vc;
  a.sel = sel;
  a.o = (__nv_bfloat16*)o;
  a.lse = lse;
  a.scores = (float*)((char*)ws + pl.scores_off);
  a.part = (float*)((char*)ws + pl.part_off);
  a.logits = logits;
  a.rule = d.select_rule;
  a.top_p = d.top_p;
  a.n_seq = d.n_seq; a.cache_len = d.cache_len; a.chunk = d.chunk; a.G = d.n_gists;
  a.top_k = d.top_k; a.window = d.window; a.Hq = d.num_q_heads; a.Hkv = d.num_kv_heads;
  a.rep = d.num_q_heads / d.num_kv_heads;
  a.n_gslices = pl.n_gslices; a.n_rslices = pl.n_rslices; a.n_part = pl.n_part;
  a.scale = d.softmax_scale > 0.f ? d.softmax_scale : 1.f / sqrtf((float)d.head_dim);
  for (int i = 0; i < 2; ++i) { a.qs[i] = d.q_strides[i]; a.os[i] = d.o_strides[i]; }
  for (int i = 0; i < 3; ++i) { a.gs[i] = d.gist_strides[i]; a.cs[i] = d.cache_strides[i]; }
  switch (a.rep) {
    case 1: return decode_launch_rep<1>(a, pl, s);
    case 2: return decode_launch_rep<2>(a, pl, s);
    case 4: return decode_launch_rep<4>(a, pl, s);
    case 8: return decode_launch_rep<8>(a, pl, s);
    default: return cudaErrorInvalidValue;
  }
}

size_t decode_workspace_bytes(const sa_decode_desc& d) { return decode_plan(d).bytes; }

// ---------------------------------------------------- gist of gists, host side
// Six launches: level-2 pass, group selection, level-1 pass over the kept
// groups, chunk selection among their level-1 gists, raw pass, combine.
struct HierPlan {
  int n2, n_cand, n_g2slices, n_cslices, n_rslices, n_part, pow2_2, pow2_1;
  size_t scores2_off, scores1_off, part_off, bytes;
};

HierPlan hier_plan(const sa_hier_decode_desc& d) {
  HierPlan p{};
  auto r256 = [](size_t x) { return (x + 255) / 256 * 256; };
  p.n2 = d.n_gists / d.fanout;
  p.n_cand = d.top_k2 * d.fanout;
  p.n_g2slices = (p.n2 + kGistSlice - 1) / kGistSlice;
  p.n_cslices = max(1, (p.n_cand + kGistSlice - 1) / kGistSlice);
  p.n_rslices = max(1, (d.top_k * d.chunk + d.window + kRawSlice - 1) / kRawSlice);
  p.n_part = p.n_g2slices + p.n_cslices + p.n_rslices;
  p.pow2_2 = 1;
  while (p.pow2_2 < p.n2) p.pow2_2 <<= 1;
  p.pow2_1 = 1;
  while (p.pow2_1 < p.n_cand) p.pow2_1 <<= 1;
  p.scores2_off = kStatusBytes;
  p.scores1_off = p.scores2_off + r256((size_t)d.n_seq * d.num_kv_heads * p.n2 * sizeof(float));
  p.part_off = p.scores1_off +
               r256((size_t)d.n_seq * d.num_kv_heads * max(p.n_cand, 1) * sizeof(float));
  p.bytes = p.part_off +
            (size_t)d.n_seq * d.num_q_heads * p.n_part * (2 + kDecD) * sizeof(float);
  return p;
}

size_t hier_decode_workspace_bytes(const sa_hier_decode_desc& d) { return hier_plan(d).bytes; }

static cudaError_t launch_select(const DecodeArgs& a, int pow2, cudaStream_t s) {
  const size_t smem = (size_t)pow2 * sizeof(unsigned long long);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(decode_select_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  decode_select_kernel<<<dim3(a.Hkv, a.n_seq), 1024, smem, s>>>(a, pow2);
  return cudaGetLastError();
}

template <int REP>
static cudaError_t hier_launch_rep(const DecodeArgs& a, const HierPlan& pl, float* scores2,
                                   float* scores1, int32_t* sel1, int top_k1, cudaStream_t s) {
  hier_gist2_kernel<REP><<<dim3(pl.n_g2slices, a.Hkv, a.n_seq), kDecThreads, 0, s>>>(a, scores2);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // groups: eligible iff all fanout * chunk raw tokens lie before the window
  DecodeArgs a2 = a;
  a2.G = a.n2;
  a2.chunk = a.fanout * a.chunk;
  a2.scores = scores2;
  a2.sel = a.sel2;
  a2.top_k = a.top_k2;
  a2.cand_groups = nullptr;
  if ((e = launch_select(a2, pl.pow2_2, s)) != cudaSuccess) return e;
  hier_gist1_kernel<REP><<<dim3(pl.n_cslices, a.Hkv, a.n_seq), kDecThreads, 0, s>>>(
      a, scores1, pl.n_g2slices);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  DecodeArgs a1 = a;
  a1.G = pl.n_cand;
  a1.scores = scores1;
  a1.sel = sel1;
  a1.top_k = top_k1;
  a1.cand_groups = a.sel2;
  if ((e = launch_select(a1, pl.pow2_1, s)) != cudaSuccess) return e;
  DecodeArgs ar = a;
  ar.sel = sel1;
  ar.top_k = top_k1;
  ar.n_gslices = pl.n_g2slices + pl.n_cslices;  // the raw partials' first slot
  decode_raw_kernel<REP><<<dim3(pl.n_rslices, a.Hkv, a.n_seq), kDecThreads, 0, s>>>(ar);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  decode_combine_kernel<<<dim3(a.Hq, a.n_seq), kDecD, 0, s>>>(a);
  return cudaGetLastError();
}

bool hier_tc_supported(const sa_hier_decode_desc& d);
cudaError_t launch_hier_decode_tc(const sa_hier_decode_desc& d, const void* q, const void* g2k,
                                  const void* g2v, const void* gk, const void* gv, const void* kc,
                                  const void* vc, int32_t* sel2, int32_t* sel1, void* o, float* lse,
                                  void* ws, cudaStream_t s);

// The tensor-core kernel (one CTA per sequence and KV head, both selections
// inside it) takes the shapes it supports; the six CUDA-core passes the rest.
cudaError_t launch_hier_decode(const sa_hier_decode_desc& d, const void* q, const void* g2k,
                               const void* g2v, const void* gk, const void* gv, const void* kc,
                               const void* vc, int32_t* sel2, int32_t* sel1, void* o, float* lse,
                               void* ws, cudaStream_t s) {
  if (hier_tc_supported(d))
    return launch_hier_decode_tc(d, q, g2k, g2v, gk, gv, kc, vc, sel2, sel1, o, lse, ws, s);
  const HierPlan pl = hier_plan(d);
  DecodeArgs a{};
  a.q = (const __nv_bfloat16*)q;
  a.g2k = (const __nv_bfloat16*)g2k;
  a.g2v = (const __nv_bfloat16*)g2v;
  a.gk = (const __nv_bfloat16*)gk;
  a.gv = (const __nv_bfloat16*)gv;
  a.kc = (const __nv_bfloat16*)kc;
  a.vc = (const __nv_bfloat16*)vc;
  a.sel2 = sel2;
  a.o = (__nv_bfloat16*)o;
  a.lse = lse;
  a.part = (float*)((char*)ws + pl.part_off);
  a.rule = SA_SELECT_SUM_LOGITS_PER_GROUP;
  a.n_seq = d.n_seq; a.cache_len = d.cache_len; a.chunk = d.chunk; a.G = d.n_gists;
  a.window = d.window; a.Hq = d.num_q_heads; a.Hkv = d.num_kv_heads;
  a.rep = d.num_q_heads / d.num_kv_heads;
  a.n2 = pl.n2; a.fanout = d.fanout; a.top_k2 = d.top_k2;
  a.n_part = pl.n_part;
  a.scale = d.softmax_scale > 0.f ? d.softmax_scale : 1.f / sqrtf((float)d.head_dim);
  for (int i = 0; i < 2; ++i) { a.qs[i] = d.q_strides[i]; a.os[i] = d.o_strides[i]; }
  for (int i = 0; i < 3; ++i) {
    a.gs[i] = d.gist_strides[i];
    a.g2s[i] = d.gist2_strides[i];
    a.cs[i] = d.cache_strides[i];
  }
  float* scores2 = (float*)((char*)ws + pl.scores2_off);
  float* scores1 = (float*)((char*)ws + pl.scores1_off);
  switch (a.rep) {
    case 1: return hier_launch_rep<1>(a, pl, scores2, scores1, sel1, d.top_k, s);
    case 2: return hier_launch_rep<2>(a, pl, scores2, scores1, sel1, d.top_k, s);
    case 4: return hier_launch_rep<4>(a, pl, scores2, scores1, sel1, d.top_k, s);
    case 8: return hier_launch_rep<8>(a, pl, scores2, scores1, sel1, d.top_k, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sa

// ---------------------------------------------------- allocation-free variant
// Scratch for sa_gist_decode_noalloc: a file-scope device array that every GPU
// loading this library holds until the process exits. All calls share it.
namespace sa {
constexpr size_t kStaticDecodeScratch = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticDecodeScratch];

constexpr int kMaxDevices = 64;
static std::mutex g_scratch_mutex;
static void* g_scratch_addr[kMaxDevices];
static CUcontext g_scratch_ctx[kMaxDevices];

// cuCtxGetCurrent through the runtime's driver entry point (no link to libcuda)
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
static CtxGetCurrentFn ctx_get_current() {
  static const CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  return fn;
}

// Device address of the array on the current device. In host code the
// array's name is only a stand-in, so the address is looked up once per device
// and context (with that device current) and cached; a new context on the
// device (after cudaDeviceReset, for one) is looked up again.
cudaError_t decode_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  CtxGetCurrentFn get = ctx_get_current();
  if (get == nullptr) return cudaErrorNotSupported;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return cudaErrorUnknown;
  if (ctx == nullptr || g_scratch_addr[dev] == nullptr || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);  // (makes the device's context current)
    if (e != cudaSuccess) return e;
    if (get(&ctx) != CUDA_SUCCESS) return cudaErrorUnknown;
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}
}  // namespace sa

extern "C" sa_status sa_gist_decode_noalloc(const sa_decode_desc* desc, const void* q,
                                            const void* gist_k, const void* gist_v,
                                            const void* k_cache, const void* v_cache,
                                            int32_t* sel_chunks, void* o, float* lse,
                                            sa_stream_t stream) {
  size_t need = 0;
  sa_status st = sa_gist_decode_workspace_size(desc, &need);  // validates the shapes
  if (st != SA_OK) return st;
  if (!(q && gist_k && gist_v && k_cache && v_cache && o && lse)) return SA_ERR_INVALID_ARG;
  if (sel_chunks == nullptr && desc->top_k != 0) return SA_ERR_INVALID_ARG;
  auto al = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; };
  if (!(al(gist_k, 16) && al(gist_v, 16) && al(k_cache, 16) && al(v_cache, 16) && al(q, 2) &&
        al(o, 2)))
    return SA_ERR_INVALID_ARG;
  if (need > sa::kStaticDecodeScratch) return SA_ERR_WORKSPACE;
  void* ws = nullptr;
  if (sa::decode_scratch_address(&ws) != cudaSuccess) return SA_ERR_CUDA;
  // the array keeps the previous call's contents: the status word must start at zero
  // (every score and partial slot is written before it is read)
  if (cudaMemsetAsync(ws, 0, sa::kStatusBytes, stream) != cudaSuccess) return SA_ERR_CUDA;
  return sa::launch_decode(*desc, q, gist_k, gist_v, k_cache, v_cache, sel_chunks, o, lse, ws,
                           stream) == cudaSuccess
             ? SA_OK
             : SA_ERR_CUDA;
}
