// CUDA-core attention kernels over the tile lists.
//
// Forward: O and LSE of softmax attention restricted to the mask, with the
// FlashAttention online softmax (running max m, running sum l, rescaled
// accumulator) over the listed 128-key tiles of each 128-query tile. This is
// the fp32 path (tensor-core tf32 would miss a 1e-5 tolerance) and the
// reference-grade path for any head_dim in {32, 64, 128}.
//
// Backward: D = rowsum(dO * O); dQ by a query-major walk over the tile CSR
// lists; dK and dV by a key-major walk over the tile CSC lists (no atomics,
// deterministic). P is recomputed from the forward's LSE.
#include "attn_mask.cuh"

namespace sa {


template <typename T>
__device__ __forceinline__ const T* row_ptr(const void* base, const int64_t* s, int bt, int pos,
                                            int h) {
  return reinterpret_cast<const T*>(base) + bt * s[0] + pos * s[1] + h * s[2];
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

// ------------------------------------------------------------------ forward
constexpr int kFwdWarps = 16;
constexpr int kFwdRows = kTile / kFwdWarps;  // query rows per warp
constexpr int kSub = 64;                     // keys staged per step

template <typename T, int D>
__global__ void __launch_bounds__(kFwdWarps * 32)
fwd_simt_kernel(AttnArgs a, MaskArgs m) {
  extern __shared__ float sm[];
  float* Qs = sm;                    // [128][D]
  float* Ks = Qs + kTile * D;        // [64][D+1]
  float* Vs = Ks + kSub * (D + 1);   // [64][D]
  const int I = blockIdx.x, h = blockIdx.y, bt = blockIdx.z;
  const int hk = h / (a.Hq / a.Hkv);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int list = list_of(m, bt, h);
  const int q0 = I * kTile;

  for (int e = threadIdx.x; e < kTile * D; e += blockDim.x) {
    const int r = e / D, c = e % D, p = q0 + r;
    Qs[e] = p < a.N ? load_as_float(row_ptr<T>(a.q, a.qs, bt, p, h) + c) : 0.f;
  }
  constexpr int C = D / 32;
  float mrow[kFwdRows], lrow[kFwdRows], acc[kFwdRows][C];
#pragma unroll
  for (int r = 0; r < kFwdRows; ++r) {
    mrow[r] = -INFINITY;
    lrow[r] = 0.f;
#pragma unroll
    for (int c = 0; c < C; ++c) acc[r][c] = 0.f;
  }

  const int e0 = m.trp[list * (m.T + 1) + I], e1 = m.trp[list * (m.T + 1) + I + 1];
  for (int e = e0; e < e1; ++e) {
    const int J = m.tcol[e];
    const bool full = m.tkind[e] == SA_TILE_FULL;
    for (int half = 0; half < kTile / kSub; ++half) {
      const int k0 = J * kTile + half * kSub;
      if (k0 >= a.N) break;
      __syncthreads();
      for (int x = threadIdx.x; x < kSub * D; x += blockDim.x) {
        const int r = x / D, c = x % D, kp = k0 + r;
        const bool ok = kp < a.N;
        Ks[r * (D + 1) + c] = ok ? load_as_float(row_ptr<T>(a.k, a.ks, bt, kp, hk) + c) : 0.f;
        Vs[r * D + c] = ok ? load_as_float(row_ptr<T>(a.v, a.vs, bt, kp, hk) + c) : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int r = 0; r < kFwdRows; ++r) {
        const int rr = warp * kFwdRows + r, p = q0 + rr;
        if (p >= a.N) continue;  // warp-uniform
        float s0 = 0.f, s1 = 0.f;
        const float* qr = Qs + rr * D;
        const float* ka = Ks + lane * (D + 1);
        const float* kb = Ks + (lane + 32) * (D + 1);
#pragma unroll 8
        for (int c = 0; c < D; ++c) {
          s0 = fmaf(qr[c], ka[c], s0);
          s1 = fmaf(qr[c], kb[c], s1);
        }
        const int kp0 = k0 + lane, kp1 = k0 + lane + 32;
        const bool v0 = kp0 < a.N && (full || element_visible(m, list, p, kp0));
        const bool v1 = kp1 < a.N && (full || element_visible(m, list, p, kp1));
        s0 = v0 ? s0 * a.scale : -INFINITY;
        s1 = v1 ? s1 * a.scale : -INFINITY;
        const float mx = warp_max(fmaxf(s0, s1));
        const float mnew = fmaxf(mrow[r], mx);
        const float ref = (mnew == -INFINITY) ? 0.f : mnew;
        const float alpha = expf(mrow[r] - ref);
        const float p0 = expf(s0 - ref), p1 = expf(s1 - ref);
        lrow[r] = lrow[r] * alpha + warp_sum(p0 + p1);
        mrow[r] = mnew;
#pragma unroll
        for (int c = 0; c < C; ++c) acc[r][c] *= alpha;
        for (int kk = 0; kk < kSub; ++kk) {
          const float pk = __shfl_sync(0xffffffffu, kk < 32 ? p0 : p1, kk & 31);
          const float* vr = Vs + kk * D + lane;
#pragma unroll
          for (int c = 0; c < C; ++c) acc[r][c] = fmaf(pk, vr[32 * c], acc[r][c]);
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kFwdRows; ++r) {
    const int p = q0 + warp * kFwdRows + r;
    if (p >= a.N) continue;
    const float inv = lrow[r] > 0.f ? 1.f / lrow[r] : 0.f;
    T* orow = const_cast<T*>(row_ptr<T>(a.o, a.os, bt, p, h));
#pragma unroll
    for (int c = 0; c < C; ++c) store_from_float(orow + lane + 32 * c, acc[r][c] * inv);
    if (lane == 0)
      a.lse[((int64_t)bt * a.Hq + h) * a.N + p] = lrow[r] > 0.f ? mrow[r] + logf(lrow[r]) : -INFINITY;
  }
}

// ----------------------------------------------------------------- backward
// D_p = sum_c dO_pc O_pc, one warp per (batch, head, row).
template <typename T, int D>
__global__ void bwd_delta_kernel(AttnArgs a) {
  const int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= (int64_t)a.Bt * a.Hq * a.N) return;
  const int p = wid % a.N, h = (wid / a.N) % a.Hq, bt = wid / ((int64_t)a.N * a.Hq);
  const T* o = row_ptr<T>(a.o, a.os, bt, p, h);
  const T* d = row_ptr<T>(a.dout, a.os, bt, p, h);
  float s = 0.f;
  for (int c = lane; c < D; c += 32) s += load_as_float(o + c) * load_as_float(d + c);
  s = warp_sum(s);
  if (lane == 0) a.delta[((int64_t)bt * a.Hq + h) * a.N + p] = s;
}

// dQ: one warp per (batch, head, query row), walking the row tile's list.
template <typename T, int D>
__global__ void bwd_dq_kernel(AttnArgs a, MaskArgs m) {
  constexpr int C = D / 32;
  const int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= (int64_t)a.Bt * a.Hq * a.N) return;
  const int p = wid % a.N, h = (wid / a.N) % a.Hq, bt = wid / ((int64_t)a.N * a.Hq);
  const int hk = h / (a.Hq / a.Hkv);
  const int list = list_of(m, bt, h);
  float qv[C], dov[C], dq[C];
  const T* qr = row_ptr<T>(a.q, a.qs, bt, p, h);
  const T* dr = row_ptr<T>(a.dout, a.os, bt, p, h);
#pragma unroll
  for (int c = 0; c < C; ++c) {
    qv[c] = load_as_float(qr + lane + 32 * c);
    dov[c] = load_as_float(dr + lane + 32 * c);
    dq[c] = 0.f;
  }
  const int64_t li = ((int64_t)bt * a.Hq + h) * a.N + p;
  const float lse = a.lse[li], Dp = a.delta[li];
  const int I = p / kTile;
  const int e0 = m.trp[list * (m.T + 1) + I], e1 = m.trp[list * (m.T + 1) + I + 1];
  for (int e = e0; e < e1; ++e) {
    const int J = m.tcol[e];
    const bool full = m.tkind[e] == SA_TILE_FULL;
    const int kend = min(a.N, (J + 1) * kTile);
    for (int kp = J * kTile; kp < kend; ++kp) {
      if (!full && !element_visible(m, list, p, kp)) continue;  // warp-uniform
      const T* kr = row_ptr<T>(a.k, a.ks, bt, kp, hk);
      const T* vr = row_ptr<T>(a.v, a.vs, bt, kp, hk);
      float s = 0.f, dp = 0.f, kv[C];
#pragma unroll
      for (int c = 0; c < C; ++c) {
        kv[c] = load_as_float(kr + lane + 32 * c);
        s = fmaf(qv[c], kv[c], s);
        dp = fmaf(dov[c], load_as_float(vr + lane + 32 * c), dp);
      }
      s = warp_sum(s);
      dp = warp_sum(dp);
      const float P = expf(s * a.scale - lse);
      const float ds = P * (dp - Dp);
#pragma unroll
      for (int c = 0; c < C; ++c) dq[c] = fmaf(ds, kv[c], dq[c]);
    }
  }
  float* out = a.dq + (((int64_t)bt * a.N + p) * a.Hq + h) * D;
#pragma unroll
  for (int c = 0; c < C; ++c) out[lane + 32 * c] = dq[c] * a.scale;
}

// dK, dV: one warp per (batch, kv head, key row), walking the key tile's
// transposed lists for every query head of the group.
template <typename T, int D>
__global__ void bwd_dkdv_kernel(AttnArgs a, MaskArgs m) {
  constexpr int C = D / 32;
  const int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= (int64_t)a.Bt * a.Hkv * a.N) return;
  const int j = wid % a.N, hk = (wid / a.N) % a.Hkv, bt = wid / ((int64_t)a.N * a.Hkv);
  const int rep = a.Hq / a.Hkv;
  float kv[C], vv[C], dk[C], dv[C];
  const T* kr = row_ptr<T>(a.k, a.ks, bt, j, hk);
  const T* vr = row_ptr<T>(a.v, a.vs, bt, j, hk);
#pragma unroll
  for (int c = 0; c < C; ++c) {
    kv[c] = load_as_float(kr + lane + 32 * c);
    vv[c] = load_as_float(vr + lane + 32 * c);
    dk[c] = 0.f;
    dv[c] = 0.f;
  }
  const int J = j / kTile;
  for (int h = hk * rep; h < (hk + 1) * rep; ++h) {
    const int list = list_of(m, bt, h);
    const int e0 = m.tcp[list * (m.T + 1) + J], e1 = m.tcp[list * (m.T + 1) + J + 1];
    for (int e = e0; e < e1; ++e) {
      const int I = m.trow[e];
      const bool full = m.tkind_t[e] == SA_TILE_FULL;
      const int pend = min(a.N, (I + 1) * kTile);
      for (int p = I * kTile; p < pend; ++p) {
        if (!full && !element_visible(m, list, p, j)) continue;  // warp-uniform
        const T* qr = row_ptr<T>(a.q, a.qs, bt, p, h);
        const T* dr = row_ptr<T>(a.dout, a.os, bt, p, h);
        float s = 0.f, dp = 0.f, qv[C], dov[C];
#pragma unroll
        for (int c = 0; c < C; ++c) {
          qv[c] = load_as_float(qr + lane + 32 * c);
          dov[c] = load_as_float(dr + lane + 32 * c);
          s = fmaf(qv[c], kv[c], s);
          dp = fmaf(dov[c], vv[c], dp);
        }
        s = warp_sum(s);
        dp = warp_sum(dp);
        const int64_t li = ((int64_t)bt * a.Hq + h) * a.N + p;
        const float P = expf(s * a.scale - a.lse[li]);
        const float ds = P * (dp - a.delta[li]);
#pragma unroll
        for (int c = 0; c < C; ++c) {
          dv[c] = fmaf(P, dov[c], dv[c]);
          dk[c] = fmaf(ds, qv[c], dk[c]);
        }
      }
    }
  }
  const int64_t o = (((int64_t)bt * a.N + j) * a.Hkv + hk) * D;
#pragma unroll
  for (int c = 0; c < C; ++c) {
    a.dk[o + lane + 32 * c] = dk[c] * a.scale;
    a.dv[o + lane + 32 * c] = dv[c];
  }
}

// ------------------------------------------------------------- host launch
template <typename T, int D>
static cudaError_t fwd_simt_launch(const AttnArgs& a, const MaskArgs& m, cudaStream_t s) {
  const size_t smem = (size_t)(kTile * D + kSub * (D + 1) + kSub * D) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(fwd_simt_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(m.T, a.Hq, a.Bt);
  fwd_simt_kernel<T, D><<<grid, kFwdWarps * 32, smem, s>>>(a, m);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t bwd_simt_launch(const AttnArgs& a, const MaskArgs& m, cudaStream_t s) {
  const int threads = 256, wpb = threads / 32;
  const int64_t nq = (int64_t)a.Bt * a.Hq * a.N, nk = (int64_t)a.Bt * a.Hkv * a.N;
  bwd_delta_kernel<T, D><<<(unsigned)((nq + wpb - 1) / wpb), threads, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_dq_kernel<T, D><<<(unsigned)((nq + wpb - 1) / wpb), threads, 0, s>>>(a, m);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_dkdv_kernel<T, D><<<(unsigned)((nk + wpb - 1) / wpb), threads, 0, s>>>(a, m);
  return cudaGetLastError();
}

cudaError_t launch_fwd_simt(int dtype, int d, const AttnArgs& a, const MaskArgs& m,
                            cudaStream_t s) {
  if (dtype == SA_DTYPE_FP32) {
    if (d == 32) return fwd_simt_launch<float, 32>(a, m, s);
    if (d == 64) return fwd_simt_launch<float, 64>(a, m, s);
    if (d == 128) return fwd_simt_launch<float, 128>(a, m, s);
  } else {
    if (d == 32) return fwd_simt_launch<__nv_bfloat16, 32>(a, m, s);
    if (d == 64) return fwd_simt_launch<__nv_bfloat16, 64>(a, m, s);
    if (d == 128) return fwd_simt_launch<__nv_bfloat16, 128>(a, m, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_simt(int dtype, int d, const AttnArgs& a, const MaskArgs& m,
                            cudaStream_t s) {
  if (dtype == SA_DTYPE_FP32) {
    if (d == 32) return bwd_simt_launch<float, 32>(a, m, s);
    if (d == 64) return bwd_simt_launch<float, 64>(a, m, s);
    if (d == 128) return bwd_simt_launch<float, 128>(a, m, s);
  } else {
    if (d == 32) return bwd_simt_launch<__nv_bfloat16, 32>(a, m, s);
    if (d == 64) return bwd_simt_launch<__nv_bfloat16, 64>(a, m, s);
    if (d == 128) return bwd_simt_launch<__nv_bfloat16, 128>(a, m, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace sa
