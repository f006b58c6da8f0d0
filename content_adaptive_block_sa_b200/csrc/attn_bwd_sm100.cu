// Block-sparse attention backward on the 5th-generation tensor cores (sm_100a).
//
// Gradients of the masked softmax attention for an upstream dO:
//   P = exp(s - LSE), dV = P^T dO, dP = dO V^T, D = rowsum(dO * O),
//   dS = P * (dP - D), dQ = dS K * scale, dK = dS^T Q * scale
// (the training use of the method: "UniGist ...", Approach, one-pass training;
// forward/backward latency is a metric that page names).
//
// One CTA per (128-key tile J, KV head, sequence) walks the transposed tile
// lists (every query tile I that visits J, for every query head of the KV
// group). TMEM lanes are key rows:
//   S^T = K_J Q_I^T and dP^T = V_J dO_I^T           (TMEM, 128 + 128 columns)
//   four compute warps form P^T and dS^T rows (bf16, swizzled shared tiles)
//   dV += P^T dO_I, dK += dS^T Q_I                   (TMEM accumulators)
//   dQ_I = dS K_J (the dS^T tile read MN-major) into the S^T columns, then
//   added to the fp32 dQ in global memory with vectorised reductions.
// A preprocess kernel writes D and LSE * log2(e) into padded workspace rows so
// that their 512-byte bulk copies never leave the buffer. All waits are
// bounded (see sm100.cuh).
#include <cuda.h>

#include "attn_mask.cuh"
#include "sm100.cuh"

namespace sa {

using namespace sm100;

struct BwdTcParams {
  CUtensorMap tmq, tmk, tmv, tmdo;
  AttnArgs a;
  MaskArgs m;
  const float* lse2;   // [Bt, Hq, Tpad] LSE * log2(e), +inf past N
  const float* delta;  // [Bt, Hq, Tpad] rowsum(dO * O), 0 past N
  int Tpad;            // T * 128
};

template <int D>
struct BwdLayout {
  static constexpr uint32_t kT = 128 * D * 2;     // a 128 x D bf16 tile
  static constexpr uint32_t kP = 128 * 128 * 2;   // a 128 x 128 bf16 tile
  static constexpr uint32_t kAtom = 128 * 128;    // [128 rows][64 bf16] swizzle atom
  static constexpr uint32_t k = 0;
  static constexpr uint32_t v = kT;
  static constexpr uint32_t q = 2 * kT;
  static constexpr uint32_t dO = 3 * kT;
  static constexpr uint32_t pt = 4 * kT;          // P^T  [keys][queries]
  static constexpr uint32_t dst = 4 * kT + kP;    // dS^T [keys][queries]
  static constexpr uint32_t rowv = 4 * kT + 2 * kP;  // lse2[128], delta[128]
  static constexpr uint32_t bars = rowv + 1024;
  static constexpr uint32_t bytes = bars + 256 + 1024;
};

enum { W_KV = 0, W_QF = 1, W_QE = 2, W_SF = 3, W_PF = 4, W_DQF = 5, W_DQE = 6, W_DRAIN = 7 };

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

template <int D>
__global__ void __launch_bounds__(192, 1) bwd_tc_kernel(const __grid_constant__ BwdTcParams P) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 16);
  volatile int* abort = reinterpret_cast<volatile int*>(bar + 16) + 1;
  float* s_lse2 = reinterpret_cast<float*>(smem + L::rowv);
  float* s_delta = s_lse2 + 128;

  const AttnArgs& a = P.a;
  const MaskArgs& m = P.m;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = m.T;
  const int hb = a.Hkv * a.Bt;
  const int J = (int)(blockIdx.x / hb);  // early key tiles (long lists) first
  const int hk = (int)(blockIdx.x % hb) % a.Hkv, bt = (int)(blockIdx.x % hb) / a.Hkv;
  const int rep = a.Hq / a.Hkv;
  const int k0 = J * kTile;
  DeviceStatus* st = a.status;

  // total visits: every query tile that lists J, for every query head of the group
  int n = 0;
  for (int r = 0; r < rep; ++r) {
    const int list = list_of(m, bt, hk * rep + r);
    n += m.tcp[list * (T + 1) + J + 1] - m.tcp[list * (T + 1) + J];
  }
  auto entry = [&](int it, int& h, int& I, int& kind) {
    for (int r = 0; r < rep; ++r) {
      const int list = list_of(m, bt, hk * rep + r);
      const int e0 = m.tcp[list * (T + 1) + J], cnt = m.tcp[list * (T + 1) + J + 1] - e0;
      if (it < cnt) {
        h = hk * rep + r;
        I = m.trow[e0 + it];
        kind = m.tkind_t[e0 + it];
        return;
      }
      it -= cnt;
    }
    h = hk * rep;
    I = 0;
    kind = SA_TILE_MASKED;
  };

  if (threadIdx.x == 0) {
    mbar_init(&bar[W_KV], 1);
    mbar_init(&bar[W_QF], 1);
    mbar_init(&bar[W_QE], 1);
    mbar_init(&bar[W_SF], 1);
    mbar_init(&bar[W_PF], 128);
    mbar_init(&bar[W_DQF], 1);
    mbar_init(&bar[W_DQE], 128);
    mbar_init(&bar[W_DRAIN], 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  constexpr uint32_t cS = 0, cDP = 128, cDV = 256, cDK = 256 + D;

  if (warp == 0) {
    if (lane == 0) {
      // -------------------------------------------------------- TMA producer
      prefetch_tmap(&P.tmq);
      prefetch_tmap(&P.tmk);
      prefetch_tmap(&P.tmv);
      prefetch_tmap(&P.tmdo);
      mbar_arrive_expect_tx(&bar[W_KV], 2 * L::kT);
      for (int at = 0; at < D / 64; ++at) {
        tma_load_4d(smem + L::k + at * L::kAtom, &P.tmk, &bar[W_KV], at * 64, hk, k0, bt);
        tma_load_4d(smem + L::v + at * L::kAtom, &P.tmv, &bar[W_KV], at * 64, hk, k0, bt);
      }
      int issued = 0;
      for (int it = 0; it < n; ++it) {
        if (!mbar_wait(&bar[W_QE], (it & 1) ^ 1, abort, st, 101)) break;
        int h, I, kind;
        entry(it, h, I, kind);
        mbar_arrive_expect_tx(&bar[W_QF], 2 * L::kT + 2 * 512);
        for (int at = 0; at < D / 64; ++at) {
          tma_load_4d(smem + L::q + at * L::kAtom, &P.tmq, &bar[W_QF], at * 64, h, I * kTile, bt);
          tma_load_4d(smem + L::dO + at * L::kAtom, &P.tmdo, &bar[W_QF], at * 64, h, I * kTile, bt);
        }
        const int64_t ro = ((int64_t)bt * a.Hq + h) * P.Tpad + (int64_t)I * kTile;
        bulk_load(s_lse2, P.lse2 + ro, 512, &bar[W_QF]);
        bulk_load(s_delta, P.delta + ro, 512, &bar[W_QF]);
        issued = it + 1;
      }
      volatile int no_abort = 0;
      mbar_wait(&bar[W_KV], 0, &no_abort, nullptr, 102);
      if (issued > 0) mbar_wait(&bar[W_QF], (issued - 1) & 1, &no_abort, nullptr, 103);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdAcc = idesc_bf16_f32(128, D, false, true);   // P^T dO, dS^T Q
      constexpr uint32_t kIdDq = idesc_bf16_f32(128, D, true, true);     // (dS^T)^T K
      bool ok = mbar_wait(&bar[W_KV], 0, abort, st, 110);
      for (int it = 0; ok && it < n; ++it) {
        if (!mbar_wait(&bar[W_QF], it & 1, abort, st, 111)) break;
        // the S^T columns hold the previous dQ until it has been read out
        if (!mbar_wait(&bar[W_DQE], (it & 1) ^ 1, abort, st, 112)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kAtom + (kk & 3) * 32;
          mma_bf16(tmem + cS, smem_desc_sw128(sb + L::k + off, 16, 1024),
                   smem_desc_sw128(sb + L::q + off, 16, 1024), kIdS, kk > 0);
          mma_bf16(tmem + cDP, smem_desc_sw128(sb + L::v + off, 16, 1024),
                   smem_desc_sw128(sb + L::dO + off, 16, 1024), kIdS, kk > 0);
        }
        mma_commit(&bar[W_SF]);
        if (!mbar_wait(&bar[W_PF], it & 1, abort, st, 113)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // K = 128 queries
          const uint32_t aoff = (kk >> 2) * L::kAtom + (kk & 3) * 32;
          mma_bf16(tmem + cDV, smem_desc_sw128(sb + L::pt + aoff, 16, 1024),
                   smem_desc_sw128(sb + L::dO + kk * 2048, L::kAtom, 1024), kIdAcc,
                   (it > 0 || kk > 0) ? 1u : 0u);
          mma_bf16(tmem + cDK, smem_desc_sw128(sb + L::dst + aoff, 16, 1024),
                   smem_desc_sw128(sb + L::q + kk * 2048, L::kAtom, 1024), kIdAcc,
                   (it > 0 || kk > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // K = 128 keys; A = dS^T read query-major
          mma_bf16(tmem + cS, smem_desc_sw128(sb + L::dst + kk * 2048, L::kAtom, 1024),
                   smem_desc_sw128(sb + L::k + kk * 2048, L::kAtom, 1024), kIdDq, kk > 0);
        mma_commit(&bar[W_DQF]);
        mma_commit(&bar[W_QE]);
      }
      mma_commit(&bar[W_DRAIN]);
      volatile int no_abort = 0;
      mbar_wait(&bar[W_DRAIN], 0, &no_abort, nullptr, 114);
    }
  } else {
    // ------------------------------------------------------- compute warps
    const int quarter = warp & 3;
    const int j = quarter * 32 + lane;  // key row of the tile = TMEM lane
    const int kq = k0 + j;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sl2 = a.scale * 1.4426950408889634f;
    const bool key_ok = kq < a.N;
    const int lb = m.b < kTile ? __ffs(m.b) - 1 : 0;
    bool ok = true;
    for (int it = 0; it < n; ++it) {
      int h, I, kind;
      entry(it, h, I, kind);
      const int list = list_of(m, bt, h);
      if (!__all_sync(0xffffffffu, mbar_wait(&bar[W_SF], it & 1, abort, st, 120))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // row-block bits of this key over the query tile (gzip, masked tiles)
      const int q0 = I * kTile;
      uint32_t qbits = 0xffffffffu;  // bit g: query block g of the tile sees this key's block
      if (kind != SA_TILE_FULL && m.b < kTile && key_ok) {
        const int kb = kq >> lb, nqb = kTile >> lb;
        qbits = 0;
        for (int g = 0; g < nqb && g < 32; ++g) {
          const int qb = (q0 >> lb) + g;
          if (qb < m.B) {
            const uint32_t* row = m.bits + ((int64_t)list * m.B + qb) * m.words;
            qbits |= ((row[kb >> 5] >> (kb & 31)) & 1u) << g;
          }
        }
      }
      uint32_t pk[64], dk[64];
      __syncwarp();  // the TMEM loads below are warp-collective (.sync.aligned)
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        float sv[32], dv[32];
        tmem_ld32(lane_addr + cS + c4 * 32, sv);
        tmem_ld32(lane_addr + cDP + c4 * 32, dv);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          float pv[2], ds[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int i = c4 * 32 + c + u;
            bool vis = key_ok;
            if (kind != SA_TILE_FULL) {
              vis = vis && kq <= q0 + i;
              if (m.b < kTile) vis = vis && ((qbits >> (i >> lb)) & 1u);
            }
            const float p = vis ? ex2(fmaf(sv[c + u], sl2, -s_lse2[i])) : 0.f;
            pv[u] = p;
            ds[u] = p * (dv[c + u] - s_delta[i]);
          }
          pk[(c4 * 32 + c) >> 1] = pack_bf16(pv[0], pv[1]);
          dk[(c4 * 32 + c) >> 1] = pack_bf16(ds[0], ds[1]);
        }
      }
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {  // rows = keys, 128 query columns
        const int col = ch * 8;
        const uint32_t off = (col >> 6) * L::kAtom + sw128_offset(j, col & 63);
        st_shared_v4(sb + L::pt + off, pk[ch * 4], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]);
        st_shared_v4(sb + L::dst + off, dk[ch * 4], dk[ch * 4 + 1], dk[ch * 4 + 2], dk[ch * 4 + 3]);
      }
      fence_async_shared();
      tc_fence_before();
      mbar_arrive(&bar[W_PF]);
      // dQ tile: TMEM lane = query row of tile I
      if (!__all_sync(0xffffffffu, mbar_wait(&bar[W_DQF], it & 1, abort, st, 121))) {
        ok = false;
        break;
      }
      tc_fence_after();
      __syncwarp();
      const int qrow = q0 + j;
      float* dq = a.dq + (((int64_t)bt * a.N + qrow) * a.Hq + h) * D;
#pragma unroll
      for (int c4 = 0; c4 < D / 32; ++c4) {
        float o[32];
        tmem_ld32(lane_addr + cS + c4 * 32, o);
        tmem_wait_ld();
        if (qrow < a.N) {
#pragma unroll
          for (int v = 0; v < 32; v += 4)
            red_add_v4(dq + c4 * 32 + v, o[v] * a.scale, o[v + 1] * a.scale, o[v + 2] * a.scale,
                       o[v + 3] * a.scale);
        }
      }
      tc_fence_before();
      mbar_arrive(&bar[W_DQE]);
    }
    // ------------------------------------------------------------- epilogue
    if (ok && n > 0) {
      // the last dQ commit follows every dV / dK MMA
      tc_fence_after();
      __syncwarp();
      float* dkr = a.dk + (((int64_t)bt * a.N + kq) * a.Hkv + hk) * D;
      float* dvr = a.dv + (((int64_t)bt * a.N + kq) * a.Hkv + hk) * D;
#pragma unroll
      for (int c4 = 0; c4 < D / 32; ++c4) {
        float x[32], y[32];
        tmem_ld32(lane_addr + cDK + c4 * 32, x);
        tmem_ld32(lane_addr + cDV + c4 * 32, y);
        tmem_wait_ld();
        if (key_ok) {
#pragma unroll
          for (int v = 0; v < 32; v += 4) {
            *reinterpret_cast<float4*>(dkr + c4 * 32 + v) =
                make_float4(x[v] * a.scale, x[v + 1] * a.scale, x[v + 2] * a.scale, x[v + 3] * a.scale);
            *reinterpret_cast<float4*>(dvr + c4 * 32 + v) = make_float4(y[v], y[v + 1], y[v + 2], y[v + 3]);
          }
        }
      }
    } else if (ok && key_ok) {
      // no query tile visits this key tile: its gradients are zero
      float* dkr = a.dk + (((int64_t)bt * a.N + kq) * a.Hkv + hk) * D;
      float* dvr = a.dv + (((int64_t)bt * a.N + kq) * a.Hkv + hk) * D;
      for (int c = 0; c < D; c += 4) {
        *reinterpret_cast<float4*>(dkr + c) = make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(dvr + c) = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// D = rowsum(dO * O) and LSE * log2(e), into padded [Bt, Hq, T*128] rows
// (+inf LSE and zero D past the end of the sequence); one warp per row.
template <int D>
__global__ void bwd_tc_prep_kernel(AttnArgs a, float* lse2, float* delta, int Tpad) {
  const int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= (int64_t)a.Bt * a.Hq * Tpad) return;
  const int p = wid % Tpad, h = (wid / Tpad) % a.Hq, bt = wid / ((int64_t)Tpad * a.Hq);
  float s = 0.f;
  if (p < a.N) {
    const __nv_bfloat16* o = reinterpret_cast<const __nv_bfloat16*>(a.o) + bt * a.os[0] +
                             (int64_t)p * a.os[1] + (int64_t)h * a.os[2];
    const __nv_bfloat16* d = reinterpret_cast<const __nv_bfloat16*>(a.dout) + bt * a.os[0] +
                             (int64_t)p * a.os[1] + (int64_t)h * a.os[2];
    for (int c = lane; c < D; c += 32) s += __bfloat162float(o[c]) * __bfloat162float(d[c]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) {
    delta[wid] = s;
    lse2[wid] = p < a.N ? a.lse[((int64_t)bt * a.Hq + h) * a.N + p] * 1.4426950408889634f
                        : INFINITY;
  }
}

// [Bt, N, H, d] bf16 with element strides {batch, seq, head}; box 64 x 1 x 128 x 1.
bool make_tile_map(CUtensorMap* map, const void* base, int d, int H, int N, int Bt,
                   const int64_t* s);

template <int D>
static cudaError_t bwd_tc_launch(const AttnArgs& a, const MaskArgs& m, void* ws, cudaStream_t s) {
  BwdTcParams P;
  memset(&P, 0, sizeof(P));
  if (!make_tile_map(&P.tmq, a.q, D, a.Hq, a.N, a.Bt, a.qs) ||
      !make_tile_map(&P.tmk, a.k, D, a.Hkv, a.N, a.Bt, a.ks) ||
      !make_tile_map(&P.tmv, a.v, D, a.Hkv, a.N, a.Bt, a.vs) ||
      !make_tile_map(&P.tmdo, a.dout, D, a.Hq, a.N, a.Bt, a.os))
    return cudaErrorInvalidValue;
  P.a = a;
  P.m = m;
  P.Tpad = m.T * kTile;
  float* lse2 = static_cast<float*>(ws);
  float* delta = lse2 + (size_t)a.Bt * a.Hq * P.Tpad;
  P.lse2 = lse2;
  P.delta = delta;
  const int64_t rows = (int64_t)a.Bt * a.Hq * P.Tpad;
  bwd_tc_prep_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(a, lse2, delta, P.Tpad);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(a.dq, 0, (size_t)a.Bt * a.N * a.Hq * D * sizeof(float), s);
  if (e != cudaSuccess) return e;
  const int bytes = (int)BwdLayout<D>::bytes;
  e = cudaFuncSetAttribute(bwd_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  bwd_tc_kernel<D><<<dim3(m.T * a.Hkv * a.Bt), 192, bytes, s>>>(P);
  return cudaGetLastError();
}

// Workspace bytes after the status header: lse2 and delta, [Bt, Hq, T*128] fp32 each.
size_t bwd_tc_workspace(int Bt, int Hq, int T) { return (size_t)2 * Bt * Hq * T * kTile * 4; }

cudaError_t launch_bwd_tc(int d, const AttnArgs& a, const MaskArgs& m, void* ws, cudaStream_t s) {
  if (d == 64) return bwd_tc_launch<64>(a, m, ws, s);
  if (d == 128) return bwd_tc_launch<128>(a, m, ws, s);
  return cudaErrorInvalidValue;
}

}  // namespace sa
