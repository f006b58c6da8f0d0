// C ABI of libsa: argument validation, size queries and dispatch.
// Every check runs on the host before any launch; a failed check returns a
// status and touches no device state.
#include <math.h>
#include <string.h>

#include "attn_mask.cuh"

namespace sa {
cudaError_t launch_gzip_build(const sa_mask_desc&, const uint8_t*, const sa_block_lists&,
                              cudaStream_t);
cudaError_t launch_gist_build(const sa_mask_desc&, const uint8_t*, const sa_block_lists&,
                              cudaStream_t);
cudaError_t launch_fwd_simt(int dtype, int d, const AttnArgs&, const MaskArgs&, cudaStream_t);
cudaError_t launch_bwd_simt(int dtype, int d, const AttnArgs&, const MaskArgs&, cudaStream_t);
cudaError_t launch_fwd_tc(int d, const AttnArgs&, const MaskArgs&, void* compact, void* near,
                          void* pair_ws, cudaStream_t);

size_t fwd_pair_workspace(int Bt, int B);
cudaError_t launch_bwd_tc(int d, const AttnArgs&, const MaskArgs&, void* ws, cudaStream_t);
size_t bwd_tc_workspace(int Bt, int Hq, int Hkv, int64_t N, int d, int T, int near_nt, bool gist);
cudaError_t launch_decode(const sa_decode_desc&, const void*, const void*, const void*,
                          const void*, const void*, int32_t*, void*, float*, void*,
                          cudaStream_t);
size_t decode_workspace_bytes(const sa_decode_desc&);
cudaError_t decode_scratch_address(void** out);
cudaError_t launch_hier_decode(const sa_hier_decode_desc&, const void*, const void*, const void*,
                               const void*, const void*, const void*, const void*, int32_t*,
                               int32_t*, void*, float*, void*, cudaStream_t);
size_t hier_decode_workspace_bytes(const sa_hier_decode_desc&);
cudaError_t launch_literal_flags_device(const uint8_t*, int, int64_t, int, uint32_t*, uint8_t*,
                                        cudaStream_t);
}  // namespace sa

using namespace sa;

#define SA_CHECK(cond, code) \
  do {                       \
    if (!(cond)) return (code); \
  } while (0)

namespace {

constexpr int64_t kMaxBlocks = 16384;
constexpr int64_t kMaxSeq = int64_t(1) << 24;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int tiles_of(int64_t n) { return (int)((n + kTile - 1) / kTile); }

// Number of lists of a mask (gzip: batch x 3 classes; gist: 1).
int64_t n_lists(const sa_mask_desc& d) { return d.kind == SA_MASK_GZIP ? (int64_t)d.batch * 3 : 1; }

// Coarse gist layout: positions per segment (raw tokens + gists); 0: fine.
int gist_period(const sa_mask_desc& d) {
  return d.kind == SA_MASK_GIST && d.block_size > 0 ? d.block_size + d.block_size / d.gist_ratio
                                                    : 0;
}

sa_status check_mask(const sa_mask_desc* d) {
  SA_CHECK(d != nullptr, SA_ERR_INVALID_ARG);
  SA_CHECK(d->seq_len >= 1 && d->seq_len <= kMaxSeq, SA_ERR_INVALID_ARG);
  SA_CHECK(d->num_heads >= 1 && d->num_heads <= kMaxHeads, SA_ERR_INVALID_ARG);
  const int64_t T = tiles_of(d->seq_len);
  if (d->kind == SA_MASK_GZIP) {
    SA_CHECK(d->batch >= 1, SA_ERR_INVALID_ARG);
    SA_CHECK(d->block_size >= 1 && d->seq_len % d->block_size == 0, SA_ERR_INVALID_ARG);
    SA_CHECK(d->block_size % kTile == 0 || kTile % d->block_size == 0, SA_ERR_UNSUPPORTED);
    SA_CHECK(d->window >= 0, SA_ERR_INVALID_ARG);
    const int64_t B = d->seq_len / d->block_size;
    SA_CHECK(B <= kMaxBlocks, SA_ERR_UNSUPPORTED);
    SA_CHECK(n_lists(*d) * (B * (B + 1) / 2) < INT32_MAX, SA_ERR_UNSUPPORTED);
    SA_CHECK(n_lists(*d) * (T * (T + 1) / 2) < INT32_MAX, SA_ERR_UNSUPPORTED);
    if (d->head_class)
      for (int h = 0; h < d->num_heads; ++h)
        SA_CHECK(d->head_class[h] >= 0 && d->head_class[h] <= 2, SA_ERR_INVALID_ARG);
    return SA_OK;
  }
  if (d->kind == SA_MASK_GIST) {
    SA_CHECK(d->batch == 1, SA_ERR_INVALID_ARG);
    SA_CHECK(d->gist_ratio >= 1 && d->sinks >= 0, SA_ERR_INVALID_ARG);
    // block_size 0: fine layout (window >= 1); > 0: coarse layout, segments
    // of block_size raw tokens and block_size / gist_ratio gists
    SA_CHECK(d->block_size >= 0 && d->block_size <= kMaxSeq, SA_ERR_INVALID_ARG);
    SA_CHECK(d->block_size > 0 ? d->block_size % d->gist_ratio == 0 : d->window >= 1,
             SA_ERR_INVALID_ARG);
    SA_CHECK(d->gist_tail == 0 || (d->gist_tail % 16 == 0 && d->gist_tail <= kTile),
             SA_ERR_INVALID_ARG);
    SA_CHECK(T * (T + 1) / 2 < INT32_MAX, SA_ERR_UNSUPPORTED);
    return SA_OK;
  }
  return SA_ERR_INVALID_ARG;
}

sa_block_lists_sizes capacity(const sa_mask_desc& d) {
  sa_block_lists_sizes c{};
  const int64_t T = tiles_of(d.seq_len), L = n_lists(d);
  c.tile_row_ptr = L * (T + 1);
  c.tile_nnz = L * T * (T + 1) / 2;
  if (d.kind == SA_MASK_GZIP) {
    const int64_t B = d.seq_len / d.block_size;
    c.row_ptr = L * (B + 1);
    c.nnz = L * B * (B + 1) / 2;
    c.bits = L * B * ((B + 31) / 32);
  } else {
    c.perm = d.seq_len;
    c.gist_bits = (d.seq_len + 31) / 32;
    c.far_idx = d.seq_len;
    c.far_ptr = T + 1;
  }
  return c;
}

sa_status check_lists(const sa_mask_desc& d, const sa_block_lists* L) {
  SA_CHECK(L != nullptr, SA_ERR_INVALID_ARG);
  const sa_block_lists_sizes c = capacity(d);
  SA_CHECK(L->tile_row_ptr && L->tile_col && L->tile_kind && L->tile_col_ptr && L->tile_row &&
               L->tile_kind_t,
           SA_ERR_INVALID_ARG);
  SA_CHECK(L->cap_tile_nnz >= c.tile_nnz, SA_ERR_WORKSPACE);
  if (d.kind == SA_MASK_GZIP) {
    SA_CHECK(L->row_ptr && L->col_idx && L->col_ptr && L->row_idx && L->bits, SA_ERR_INVALID_ARG);
    SA_CHECK(L->cap_nnz >= c.nnz, SA_ERR_WORKSPACE);
  } else {
    SA_CHECK(L->perm && L->gist_bits && L->far_idx && L->far_ptr, SA_ERR_INVALID_ARG);
  }
  return SA_OK;
}

sa_status check_ws(void* ws, size_t have, size_t need) {
  SA_CHECK(ws != nullptr && aligned(ws, 256), SA_ERR_INVALID_ARG);
  SA_CHECK(have >= need, SA_ERR_WORKSPACE);
  return SA_OK;
}

sa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SA_OK : SA_ERR_CUDA; }

sa_status clear_status(void* ws, cudaStream_t s) {
  return cuda_status(cudaMemsetAsync(ws, 0, kStatusBytes, s));
}

sa_status check_attn(const sa_attn_desc* a, const sa_mask_desc* m) {
  SA_CHECK(a != nullptr, SA_ERR_INVALID_ARG);
  sa_status st = check_mask(m);
  if (st != SA_OK) return st;
  SA_CHECK(a->dtype == SA_DTYPE_BF16 || a->dtype == SA_DTYPE_FP32, SA_ERR_INVALID_ARG);
  SA_CHECK(a->batch >= 1 && a->seq_len == m->seq_len, SA_ERR_INVALID_ARG);
  if (m->kind == SA_MASK_GZIP) SA_CHECK(a->batch == m->batch, SA_ERR_INVALID_ARG);
  SA_CHECK(a->num_q_heads == m->num_heads, SA_ERR_INVALID_ARG);
  SA_CHECK(a->num_kv_heads >= 1 && a->num_q_heads % a->num_kv_heads == 0, SA_ERR_INVALID_ARG);
  SA_CHECK(a->head_dim == 32 || a->head_dim == 64 || a->head_dim == 128, SA_ERR_UNSUPPORTED);
  SA_CHECK(a->softmax_scale >= 0.f && isfinite(a->softmax_scale), SA_ERR_INVALID_ARG);
  SA_CHECK(a->impl >= SA_IMPL_AUTO && a->impl <= SA_IMPL_TENSOR_CORES, SA_ERR_INVALID_ARG);
  const int64_t* all[4] = {a->q_strides, a->k_strides, a->v_strides, a->o_strides};
  for (auto s : all) {
    SA_CHECK(s[0] >= 0 && s[2] >= 0 && s[1] >= a->head_dim, SA_ERR_INVALID_ARG);
  }
  return SA_OK;
}

MaskArgs make_mask_args(const sa_mask_desc& d, const sa_block_lists& L) {
  MaskArgs m{};
  m.kind = d.kind;
  m.T = tiles_of(d.seq_len);
  m.trp = L.tile_row_ptr;
  m.tcol = L.tile_col;
  m.tkind = L.tile_kind;
  m.tcp = L.tile_col_ptr;
  m.trow = L.tile_row;
  m.tkind_t = L.tile_kind_t;
  if (d.kind == SA_MASK_GZIP) {
    m.bits = L.bits;
    m.b = d.block_size;
    m.B = (int)(d.seq_len / d.block_size);
    m.words = (m.B + 31) / 32;
    m.wb = d.window;
    const int H = d.num_heads, n_loc = H / 2, n_lit = H / 4;
    for (int h = 0; h < H; ++h)
      m.head_class[h] = d.head_class ? (uint8_t)d.head_class[h]
                                     : (uint8_t)(h < n_loc ? SA_CLASS_LOCAL
                                                 : h < n_loc + n_lit ? SA_CLASS_LITERAL
                                                                     : SA_CLASS_HYBRID);
  } else {
    m.perm = L.perm;
    m.gist_bits = L.gist_bits;
    m.far_idx = L.far_idx;
    m.far_ptr = L.far_ptr;
    m.sinks = d.sinks;
    m.window = d.window;
    m.period = gist_period(d);
  }
  return m;
}

AttnArgs make_attn_args(const sa_attn_desc& a) {
  AttnArgs r{};
  r.Bt = a.batch;
  r.N = (int)a.seq_len;
  r.Hq = a.num_q_heads;
  r.Hkv = a.num_kv_heads;
  r.scale = a.softmax_scale > 0.f ? a.softmax_scale : 1.f / sqrtf((float)a.head_dim);
  for (int i = 0; i < 3; ++i) {
    r.qs[i] = a.q_strides[i];
    r.ks[i] = a.k_strides[i];
    r.vs[i] = a.v_strides[i];
    r.os[i] = a.o_strides[i];
  }
  return r;
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Can the TMA + tcgen05 kernels read these tensors?
bool tensor_core_ok(const sa_attn_desc& a, const void* const* ptrs, int nptr) {
  if (a.dtype != SA_DTYPE_BF16 || (a.head_dim != 64 && a.head_dim != 128)) return false;
  for (int i = 0; i < nptr; ++i)
    if (!aligned(ptrs[i], 16)) return false;
  const int64_t* all[4] = {a.q_strides, a.k_strides, a.v_strides, a.o_strides};
  for (auto s : all)
    for (int i = 0; i < 3; ++i)
      if (s[i] % 8 != 0) return false;
  return true;
}

// Resolves SA_IMPL_AUTO; -1 if the request cannot be served.
int pick_impl(const sa_attn_desc& a, bool tc_ok) {
  if (a.impl == SA_IMPL_AUTO) return tc_ok ? SA_IMPL_TENSOR_CORES : SA_IMPL_CUDA_CORES;
  if (a.impl == SA_IMPL_TENSOR_CORES && !tc_ok) return -1;
  return a.impl;
}

}  // namespace

extern "C" {

const char* sa_version(void) { return "0.1.0 (sm_100a)"; }

const char* sa_status_string(sa_status st) {
  switch (st) {
    case SA_OK: return "SA_OK";
    case SA_ERR_INVALID_ARG: return "SA_ERR_INVALID_ARG";
    case SA_ERR_UNSUPPORTED: return "SA_ERR_UNSUPPORTED";
    case SA_ERR_WORKSPACE: return "SA_ERR_WORKSPACE";
    case SA_ERR_CUDA: return "SA_ERR_CUDA";
    case SA_ERR_TIMEOUT: return "SA_ERR_TIMEOUT";
    case SA_ERR_DEVICE: return "SA_ERR_DEVICE";
  }
  return "SA_UNKNOWN_STATUS";
}

sa_status sa_get_device_status(const void* ws, sa_stream_t stream, sa_status* out) {
  SA_CHECK(out != nullptr, SA_ERR_INVALID_ARG);
  if (ws == nullptr) {  // the allocation-free decode's fixed scratch array
    void* p = nullptr;
    if (decode_scratch_address(&p) != cudaSuccess) return SA_ERR_CUDA;
    ws = p;
  }
  int32_t code = 0;
  cudaError_t e = cudaMemcpyAsync(&code, ws, sizeof(code), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return SA_ERR_CUDA;
  *out = (sa_status)code;
  return SA_OK;
}

sa_status sa_literal_flags_from_sizes(const uint32_t* sizes, int32_t num_blocks, uint8_t* flags) {
  SA_CHECK(sizes != nullptr && flags != nullptr && num_blocks >= 1, SA_ERR_INVALID_ARG);
  uint64_t total = 0;
  for (int32_t i = 0; i < num_blocks; ++i) total += sizes[i];
  for (int32_t i = 0; i < num_blocks; ++i)
    flags[i] = (uint64_t)sizes[i] * (uint64_t)num_blocks > total ? 1 : 0;
  return SA_OK;
}

sa_status sa_block_lists_capacity(const sa_mask_desc* desc, sa_block_lists_sizes* out) {
  sa_status st = check_mask(desc);
  if (st != SA_OK) return st;
  SA_CHECK(out != nullptr, SA_ERR_INVALID_ARG);
  *out = capacity(*desc);
  return SA_OK;
}

sa_status sa_build_block_mask_workspace_size(const sa_mask_desc* desc, size_t* bytes) {
  sa_status st = check_mask(desc);
  if (st != SA_OK) return st;
  SA_CHECK(bytes != nullptr, SA_ERR_INVALID_ARG);
  *bytes = kStatusBytes;
  return SA_OK;
}

sa_status sa_literal_flags_device(const uint8_t* bytes, int32_t batch, int64_t n_bytes,
                                  int32_t block_bytes, uint32_t* sizes, uint8_t* flags,
                                  sa_stream_t stream) {
  SA_CHECK(bytes && sizes && flags, SA_ERR_INVALID_ARG);
  SA_CHECK(batch >= 1 && n_bytes >= 1, SA_ERR_INVALID_ARG);
  SA_CHECK(block_bytes >= 1 && n_bytes % block_bytes == 0, SA_ERR_INVALID_ARG);
  SA_CHECK(block_bytes <= 1024, SA_ERR_UNSUPPORTED);
  SA_CHECK(n_bytes / block_bytes <= kMaxBlocks, SA_ERR_UNSUPPORTED);
  SA_CHECK(aligned(sizes, 4), SA_ERR_INVALID_ARG);
  return cuda_status(launch_literal_flags_device(bytes, batch, n_bytes, block_bytes, sizes, flags,
                                                 (cudaStream_t)stream));
}

sa_status sa_build_block_mask(const sa_mask_desc* desc, const uint8_t* d_flags,
                              const sa_block_lists* out, void* ws, size_t ws_bytes,
                              sa_stream_t stream) {
  sa_status st = check_mask(desc);
  if (st != SA_OK) return st;
  if (desc->kind == SA_MASK_GZIP) SA_CHECK(d_flags != nullptr, SA_ERR_INVALID_ARG);
  // the coarse gist layout takes its regular pattern only
  if (desc->kind == SA_MASK_GIST && desc->block_size > 0)
    SA_CHECK(d_flags == nullptr, SA_ERR_INVALID_ARG);
  st = check_lists(*desc, out);
  if (st != SA_OK) return st;
  st = check_ws(ws, ws_bytes, kStatusBytes);
  if (st != SA_OK) return st;
  st = clear_status(ws, stream);
  if (st != SA_OK) return st;
  cudaError_t e = desc->kind == SA_MASK_GZIP ? launch_gzip_build(*desc, d_flags, *out, stream)
                                             : launch_gist_build(*desc, d_flags, *out, stream);
  return cuda_status(e);
}

// The tensor-core forward pairs 64-token query blocks into 128-row tiles
// (b = 64; block indices must fit the 12-bit fields of its visit entries).
static bool pair_mode(const sa_mask_desc& m) {
  return m.kind == SA_MASK_GZIP && m.block_size == 64 && m.seq_len / 64 <= 4094;
}

sa_status sa_forward_workspace_size(const sa_attn_desc* attn, const sa_mask_desc* mask,
                                    size_t* bytes) {
  sa_status st = check_attn(attn, mask);
  if (st != SA_OK) return st;
  SA_CHECK(bytes != nullptr, SA_ERR_INVALID_ARG);
  *bytes = kStatusBytes;
  if (pair_mode(*mask)) *bytes += fwd_pair_workspace(mask->batch, (int)(mask->seq_len / 64));
  if (mask->kind == SA_MASK_GIST) {
    // tensor-core path: compacted sink/gist K and V, then the element masks of
    // every (query tile, near key tile) pair, 128 x 128 bits each
    *bytes += 2 * round256((size_t)attn->batch * attn->seq_len * attn->num_kv_heads *
                           attn->head_dim * 2);
    *bytes += round256((size_t)tiles_of(attn->seq_len) *
                       gist_near_tiles(mask->window, gist_period(*mask)) * 2048);
  }
  return SA_OK;
}

sa_status sa_forward(const sa_attn_desc* attn, const sa_mask_desc* mask, const void* q,
                     const void* k, const void* v, const sa_block_lists* lists, void* o,
                     float* lse, void* ws, size_t ws_bytes, sa_stream_t stream) {
  sa_status st = check_attn(attn, mask);
  if (st != SA_OK) return st;
  SA_CHECK(q && k && v && o && lse, SA_ERR_INVALID_ARG);
  const size_t esz = attn->dtype == SA_DTYPE_BF16 ? 2 : 4;
  SA_CHECK(aligned(q, esz) && aligned(k, esz) && aligned(v, esz) && aligned(o, esz) &&
               aligned(lse, 4),
           SA_ERR_INVALID_ARG);
  st = check_lists(*mask, lists);
  if (st != SA_OK) return st;
  size_t need = 0;
  sa_forward_workspace_size(attn, mask, &need);
  st = check_ws(ws, ws_bytes, need);
  if (st != SA_OK) return st;
  AttnArgs a = make_attn_args(*attn);
  a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
  a.status = (DeviceStatus*)ws;
  const void* ptrs[4] = {q, k, v, o};
  const int impl = pick_impl(*attn, tensor_core_ok(*attn, ptrs, 4));
  if (impl < 0) return SA_ERR_UNSUPPORTED;
  st = clear_status(ws, stream);
  if (st != SA_OK) return st;
  const MaskArgs m = make_mask_args(*mask, *lists);
  if (impl == SA_IMPL_TENSOR_CORES) {
    char* compact = (char*)ws + kStatusBytes;
    char* near = compact + 2 * round256((size_t)attn->batch * attn->seq_len *
                                        attn->num_kv_heads * attn->head_dim * 2);
    void* pair_ws = pair_mode(*mask) ? (char*)ws + kStatusBytes : nullptr;
    return cuda_status(launch_fwd_tc(attn->head_dim, a, m, compact, near, pair_ws, stream));
  }
  return cuda_status(launch_fwd_simt(attn->dtype, attn->head_dim, a, m, stream));
}

sa_status sa_backward_workspace_size(const sa_attn_desc* attn, const sa_mask_desc* mask,
                                     size_t* bytes) {
  sa_status st = check_attn(attn, mask);
  if (st != SA_OK) return st;
  SA_CHECK(bytes != nullptr, SA_ERR_INVALID_ARG);
  const size_t simt = (size_t)attn->batch * attn->num_q_heads * attn->seq_len * sizeof(float);
  const size_t tc = bwd_tc_workspace(attn->batch, attn->num_q_heads, attn->num_kv_heads,
                                     attn->seq_len, attn->head_dim, tiles_of(attn->seq_len),
                                     gist_near_tiles(mask->window, gist_period(*mask)),
                                     mask->kind == SA_MASK_GIST);
  *bytes = kStatusBytes + round256(simt > tc ? simt : tc);
  return SA_OK;
}

sa_status sa_backward(const sa_attn_desc* attn, const sa_mask_desc* mask, const void* q,
                      const void* k, const void* v, const void* o, const float* lse,
                      const void* dout, const sa_block_lists* lists, float* dq, float* dk,
                      float* dv, void* ws, size_t ws_bytes, sa_stream_t stream) {
  size_t need = 0;
  sa_status st = sa_backward_workspace_size(attn, mask, &need);
  if (st != SA_OK) return st;
  SA_CHECK(q && k && v && o && lse && dout && dq && dk && dv, SA_ERR_INVALID_ARG);
  SA_CHECK(aligned(dq, 4) && aligned(dk, 4) && aligned(dv, 4), SA_ERR_INVALID_ARG);
  st = check_lists(*mask, lists);
  if (st != SA_OK) return st;
  st = check_ws(ws, ws_bytes, need);
  if (st != SA_OK) return st;
  // tensor cores: bf16, gzip masks with b >= 4 or the gist layout (fp32
  // inputs use the CUDA-core kernels)
  const void* ptrs[5] = {q, k, v, o, dout};
  const bool tc_ok = tensor_core_ok(*attn, ptrs, 5) &&
                     (mask->kind == SA_MASK_GIST || mask->block_size >= 4) && aligned(dq, 16) &&
                     aligned(dk, 16) && aligned(dv, 16);
  const int impl = pick_impl(*attn, tc_ok);
  if (impl < 0) return SA_ERR_UNSUPPORTED;
  st = clear_status(ws, stream);
  if (st != SA_OK) return st;
  AttnArgs a = make_attn_args(*attn);
  a.q = q; a.k = k; a.v = v; a.o = const_cast<void*>(o); a.lse = const_cast<float*>(lse);
  a.dout = dout; a.dq = dq; a.dk = dk; a.dv = dv;
  a.delta = (float*)((char*)ws + kStatusBytes);
  a.status = (DeviceStatus*)ws;
  const MaskArgs m = make_mask_args(*mask, *lists);
  if (impl == SA_IMPL_TENSOR_CORES)
    return cuda_status(launch_bwd_tc(attn->head_dim, a, m, (char*)ws + kStatusBytes, stream));
  return cuda_status(launch_bwd_simt(attn->dtype, attn->head_dim, a, m, stream));
}

static sa_status check_decode(const sa_decode_desc* d) {
  SA_CHECK(d != nullptr, SA_ERR_INVALID_ARG);
  SA_CHECK(d->n_seq >= 1 && d->chunk >= 1 && d->n_gists >= 1, SA_ERR_INVALID_ARG);
  SA_CHECK((int64_t)d->n_gists * d->chunk == d->cache_len, SA_ERR_INVALID_ARG);
  SA_CHECK(d->n_gists <= 8192, SA_ERR_UNSUPPORTED);
  SA_CHECK(d->top_k >= 0 && d->top_k <= 256, SA_ERR_UNSUPPORTED);
  SA_CHECK(d->window >= 0 && d->window <= d->cache_len, SA_ERR_INVALID_ARG);
  SA_CHECK(d->num_kv_heads >= 1 && d->num_q_heads % d->num_kv_heads == 0, SA_ERR_INVALID_ARG);
  const int rep = d->num_q_heads / d->num_kv_heads;
  SA_CHECK(rep == 1 || rep == 2 || rep == 4 || rep == 8, SA_ERR_UNSUPPORTED);
  SA_CHECK(d->head_dim == 128, SA_ERR_UNSUPPORTED);
  SA_CHECK(d->select_rule >= SA_SELECT_SUM_LOGITS_PER_GROUP &&
               d->select_rule <= SA_SELECT_TOP_K_PER_HEAD,
           SA_ERR_INVALID_ARG);
  if (d->select_rule == SA_SELECT_TOP_P_PER_GROUP)
    SA_CHECK(d->top_p > 0.f && d->top_p <= 1.f, SA_ERR_INVALID_ARG);
  SA_CHECK(d->softmax_scale >= 0.f && isfinite(d->softmax_scale), SA_ERR_INVALID_ARG);
  // 16-byte row loads
  SA_CHECK(d->gist_strides[2] % 8 == 0 && d->cache_strides[2] % 8 == 0, SA_ERR_INVALID_ARG);
  SA_CHECK(d->gist_strides[0] % 8 == 0 && d->gist_strides[1] % 8 == 0, SA_ERR_INVALID_ARG);
  SA_CHECK(d->cache_strides[0] % 8 == 0 && d->cache_strides[1] % 8 == 0, SA_ERR_INVALID_ARG);
  return SA_OK;
}

sa_status sa_gist_decode_workspace_size(const sa_decode_desc* desc, size_t* bytes) {
  sa_status st = check_decode(desc);
  if (st != SA_OK) return st;
  SA_CHECK(bytes != nullptr, SA_ERR_INVALID_ARG);
  *bytes = decode_workspace_bytes(*desc);
  return SA_OK;
}

sa_status sa_gist_decode(const sa_decode_desc* desc, const void* q, const void* gist_k,
                         const void* gist_v, const void* k_cache, const void* v_cache,
                         int32_t* sel_chunks, void* o, float* lse, void* ws, size_t ws_bytes,
                         sa_stream_t stream) {
  size_t need = 0;
  sa_status st = sa_gist_decode_workspace_size(desc, &need);
  if (st != SA_OK) return st;
  SA_CHECK(q && gist_k && gist_v && k_cache && v_cache && o && lse, SA_ERR_INVALID_ARG);
  SA_CHECK(sel_chunks != nullptr || desc->top_k == 0, SA_ERR_INVALID_ARG);
  SA_CHECK(aligned(gist_k, 16) && aligned(gist_v, 16) && aligned(k_cache, 16) &&
               aligned(v_cache, 16) && aligned(q, 2) && aligned(o, 2),
           SA_ERR_INVALID_ARG);
  st = check_ws(ws, ws_bytes, need);
  if (st != SA_OK) return st;
  st = clear_status(ws, stream);
  if (st != SA_OK) return st;
  return cuda_status(launch_decode(*desc, q, gist_k, gist_v, k_cache, v_cache, sel_chunks, o,
                                   lse, ws, stream));
}

static sa_status check_hier_decode(const sa_hier_decode_desc* d) {
  SA_CHECK(d != nullptr, SA_ERR_INVALID_ARG);
  SA_CHECK(d->n_seq >= 1 && d->chunk >= 1 && d->fanout >= 1 && d->n_gists >= 1,
           SA_ERR_INVALID_ARG);
  SA_CHECK(d->n_gists % d->fanout == 0, SA_ERR_INVALID_ARG);
  SA_CHECK((int64_t)d->n_gists * d->chunk == d->cache_len, SA_ERR_INVALID_ARG);
  SA_CHECK(d->n_gists / d->fanout <= 8192, SA_ERR_UNSUPPORTED);
  SA_CHECK(d->top_k2 >= 0 && d->top_k2 <= 256 && d->top_k >= 0 && d->top_k <= 256,
           SA_ERR_UNSUPPORTED);
  SA_CHECK((int64_t)d->top_k2 * d->fanout <= 8192, SA_ERR_UNSUPPORTED);
  SA_CHECK(d->window >= 0 && d->window <= d->cache_len, SA_ERR_INVALID_ARG);
  SA_CHECK(d->num_kv_heads >= 1 && d->num_q_heads % d->num_kv_heads == 0, SA_ERR_INVALID_ARG);
  const int rep = d->num_q_heads / d->num_kv_heads;
  SA_CHECK(rep == 1 || rep == 2 || rep == 4 || rep == 8, SA_ERR_UNSUPPORTED);
  SA_CHECK(d->head_dim == 128, SA_ERR_UNSUPPORTED);
  SA_CHECK(d->softmax_scale >= 0.f && isfinite(d->softmax_scale), SA_ERR_INVALID_ARG);
  for (int i = 0; i < 3; ++i)  // 16-byte row loads
    SA_CHECK(d->gist_strides[i] % 8 == 0 && d->gist2_strides[i] % 8 == 0 &&
                 d->cache_strides[i] % 8 == 0,
             SA_ERR_INVALID_ARG);
  return SA_OK;
}

sa_status sa_gist_hier_decode_workspace_size(const sa_hier_decode_desc* desc, size_t* bytes) {
  sa_status st = check_hier_decode(desc);
  if (st != SA_OK) return st;
  SA_CHECK(bytes != nullptr, SA_ERR_INVALID_ARG);
  *bytes = hier_decode_workspace_bytes(*desc);
  return SA_OK;
}

sa_status sa_gist_hier_decode(const sa_hier_decode_desc* desc, const void* q, const void* gist2_k,
                              const void* gist2_v, const void* gist_k, const void* gist_v,
                              const void* k_cache, const void* v_cache, int32_t* sel_groups,
                              int32_t* sel_chunks, void* o, float* lse, void* ws,
                              size_t ws_bytes, sa_stream_t stream) {
  size_t need = 0;
  sa_status st = sa_gist_hier_decode_workspace_size(desc, &need);
  if (st != SA_OK) return st;
  SA_CHECK(q && gist2_k && gist2_v && gist_k && gist_v && k_cache && v_cache && o && lse,
           SA_ERR_INVALID_ARG);
  SA_CHECK(sel_groups != nullptr || desc->top_k2 == 0, SA_ERR_INVALID_ARG);
  SA_CHECK(sel_chunks != nullptr || desc->top_k == 0, SA_ERR_INVALID_ARG);
  SA_CHECK(aligned(gist2_k, 16) && aligned(gist2_v, 16) && aligned(gist_k, 16) &&
               aligned(gist_v, 16) && aligned(k_cache, 16) && aligned(v_cache, 16) &&
               aligned(q, 2) && aligned(o, 2),
           SA_ERR_INVALID_ARG);
  st = check_ws(ws, ws_bytes, need);
  if (st != SA_OK) return st;
  st = clear_status(ws, stream);
  if (st != SA_OK) return st;
  return cuda_status(launch_hier_decode(*desc, q, gist2_k, gist2_v, gist_k, gist_v, k_cache,
                                        v_cache, sel_groups, sel_chunks, o, lse, ws, stream));
}

}  // extern "C"
