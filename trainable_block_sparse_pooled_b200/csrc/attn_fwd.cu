// Block-sparse attention forward on sm_100a: step 4 of SpargeAttention2
// (paper.rainbus.top summary, 方法步骤详情 step 4; 前置知识 "稀疏注意力" and
// "块稀疏注意力": masked Q_i K_j^T and P_ij V_j tiles are skipped; gist.science 2C).
//
// One CTA per (q-block i, head): 128 query rows (b_q = 128) against the kept
// kv-blocks j (b_kv = 64 rows each) listed in the CSR row of i.
//
//   warp 4      TMA producer: Q_i once, then K_j and V_j through 2-slot rings;
//               a K slot is refilled as soon as its S product is done, a V slot
//               once its P V product is done (whichever is free first).
//   warp 5      MMA issuer (all 32 lanes run the loop, elect.sync picks the lane
//               that issues each tcgen05 op): S = Q K_j^T (SS, bf16, M=128 N=64 K=d)
//               into one of two TMEM S buffers; O += P V_j (TS: P from TMEM,
//               fp16 operands, M=128 N=d K=64). Owns the 256-column TMEM
//               allocation.
//   warps 0-3   softmax, thread t <-> query row t <-> TMEM lane t: load S,
//               online max / exp2 / sum in registers, write P (fp16, values in
//               [0, 256]: 8x finer rounding than bf16) over the S buffer,
//               rescale O in TMEM only when the running max grew by more than
//               2^8 (lazy rescale), then the epilogue O / l -> bf16
//               (and optionally its bf16 residual) -> smem -> TMA store, LSE.
//
// TMEM columns: [0,64) S/P buffer 0, [64,128) S/P buffer 1, [128,128+d) O.
// v_to_f16_kernel  fp16 copy of V for the P V product (exact for bf16 values
//               of magnitude <= 65504; larger ones are clamped and reported).
// Shared memory: Q 128 x d bf16 (reused as the O staging tile), 2 x (K bf16,
// V fp16) 64 x d; every tile in 128-byte-swizzled 64-column chunks as TMA writes
// them. Two CTAs fit on one SM (TMEM 2 x 256 columns, smem 2 x ~97 KB), so one
// CTA's softmax overlaps the other's MMAs.
#include "common.cuh"
#include "kernels.h"

namespace spa2 {

namespace {

template <int D>
struct FwdSmem {
  static constexpr int CH = D / 64;  // 64-column chunks per row
  alignas(1024) uint8_t q[CH][128 * 128];
  alignas(1024) uint8_t k[2][CH][64 * 128];
  alignas(1024) uint8_t v[2][CH][64 * 128];
  uint64_t q_full;
  uint64_t k_full[2], v_full[2], k_empty[2], v_empty[2];
  uint64_t s_full[2], p_full[2], o_done, drain;
  uint32_t tmem_base;
  int abort_flag;
  int epi_ok;
  int never;  // stays 0: abort flag of the teardown drains
};

SPA2_DEV bool wait_warp(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  const bool ok = wait_bar(bar, parity, w);
  return __all_sync(0xffffffff, ok);
}

}  // namespace

// TILED: the list entries may carry exclusion bits (block sizes other than
// (128, 64)); without it they are plain ids and no check is compiled in
template <int D, bool TILED>
__global__ void __launch_bounds__(192, 2) fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                     const __grid_constant__ CUtensorMap tm_k,
                                                     const __grid_constant__ CUtensorMap tm_v,
                                                     const __grid_constant__ CUtensorMap tm_o,
                                                     const __grid_constant__ CUtensorMap tm_olo, int has_olo,
                                                     const int* __restrict__ row_cnt, const int* __restrict__ row_idx,
                                                     float* __restrict__ lse, int N, int Tm, int Tn, float scale_log2,
                                                     int* status, unsigned long long wait_limit_ns) {
  constexpr int CH = D / 64;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64, false, false);
  constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, false, true, /*f16=*/true);
  constexpr uint32_t Q_BYTES = 128 * D * 2;
  constexpr uint32_t KV_BYTES = 64 * D * 2;

  extern __shared__ uint8_t smem_raw[];
  FwdSmem<D>& sm = *reinterpret_cast<FwdSmem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 5), 0);  // warp-uniform
  const uint32_t lane = lane_id();
  const int i = blockIdx.x;
  const int bh = blockIdx.y;
  const long long rowid = (long long)bh * Tm + i;

  if (warp == 5) {
    tmem_alloc(&sm.tmem_base, 256);
    tmem_relinquish();
  }
  if (threadIdx.x == 128) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
      mbar_init(&sm.v_empty[s], 1);
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], 128);
    }
    mbar_init(&sm.o_done, 1);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    sm.epi_ok = 0;
    sm.never = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const WaitCtx wc{&sm.abort_flag, status, wait_limit_ns};

  int n = __shfl_sync(0xffffffffu, row_cnt[rowid], 0);  // warp-uniform
  if (n < 1 || n > Tn) {
    if (threadIdx.x == 0) report(status, SPA2_ERR_DEVICE_BOUNDS);
    n = 0;
  }
  const int* kv_list = row_idx + rowid * Tn;

  if (warp == 4) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && n > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_expect_tx(&sm.q_full, Q_BYTES);
      for (int c = 0; c < CH; ++c) tma_load_3d(sm.q[c], &tm_q, &sm.q_full, c * 64, i * 128, bh);
      // the fp16 copy of V comes from the kernel launched just before this one
      pdl_wait();
      // K(kt) needs S(kt - 2) done, V(vt) needs P V(vt - 2) done; take whichever
      // is free, K first (its product comes first)
      int kt = 0, vt = 0;
      uint64_t t0 = 0;
      uint32_t idle = 0;
      while (vt < n) {
        if (kt < n && (kt < 2 || mbar_test_wait(&sm.k_empty[kt & 1], ((kt >> 1) - 1) & 1))) {
          const int j = kv_list[kt] & TILE_ID_MASK;
          if (j >= Tn) {
            report(status, SPA2_ERR_DEVICE_BOUNDS);
            sm.abort_flag = 1;
            break;
          }
          mbar_expect_tx(&sm.k_full[kt & 1], KV_BYTES);
          for (int c = 0; c < CH; ++c) tma_load_3d(sm.k[kt & 1][c], &tm_k, &sm.k_full[kt & 1], c * 64, j * 64, bh);
          ++kt;
          idle = 0;
          t0 = 0;
        } else if (vt < kt && (vt < 2 || mbar_test_wait(&sm.v_empty[vt & 1], ((vt >> 1) - 1) & 1))) {
          const int j = kv_list[vt] & TILE_ID_MASK;
          mbar_expect_tx(&sm.v_full[vt & 1], KV_BYTES);
          for (int c = 0; c < CH; ++c) tma_load_3d(sm.v[vt & 1][c], &tm_v, &sm.v_full[vt & 1], c * 64, j * 64, bh);
          ++vt;
          idle = 0;
          t0 = 0;
        } else {
          // nothing free: sleep in try_wait on the slot that frees next, not a hot spin
          if (kt < n && kt >= 2)
            mbar_try_wait(&sm.k_empty[kt & 1], ((kt >> 1) - 1) & 1);
          else if (vt < kt && vt >= 2)
            mbar_try_wait(&sm.v_empty[vt & 1], ((vt >> 1) - 1) & 1);
          if ((++idle & 63u) != 0u) continue;
          if (sm.abort_flag) break;
          const uint64_t now = globaltimer_ns();
          if (t0 == 0) {
            t0 = now;
          } else if (now - t0 > wait_limit_ns) {
            report(status, SPA2_ERR_DEVICE_TIMEOUT);
            sm.abort_flag = 1;
            break;
          }
        }
      }
      // never leave with copies in flight: wait (bounded) for the last loads
      const WaitCtx drain_wc{&sm.never, nullptr, wait_limit_ns};
      for (int t = max(0, kt - 2); t < kt; ++t) wait_bar(&sm.k_full[t & 1], (t >> 1) & 1, drain_wc);
      for (int t = max(0, vt - 2); t < vt; ++t) wait_bar(&sm.v_full[t & 1], (t >> 1) & 1, drain_wc);
      wait_bar(&sm.q_full, 0, drain_wc);
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer ----------------
    if (n > 0) {  // all 32 lanes; elect.sync picks the issuing lane
      const uint32_t tmem_o = tmem + 128;
      if (wait_bar_all(&sm.q_full, 0, wc)) {
        for (int t = 0; t <= n; ++t) {
          if (t < n) {
            const int s = t & 1;
            if (!wait_bar_all(&sm.k_full[s], (t >> 1) & 1, wc)) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t a = sdesc_sw128(smem_u32(sm.q[kk >> 2]) + (kk & 3) * 32, 16, 1024);
              const uint64_t b = sdesc_sw128(smem_u32(sm.k[s][kk >> 2]) + (kk & 3) * 32, 16, 1024);
              mma_ss_el(tmem + s * 64, a, b, IDESC_S, kk > 0 ? 1u : 0u);
            }
            mma_commit_el(&sm.s_full[s]);
            mma_commit_el(&sm.k_empty[s]);
          }
          if (t >= 1) {
            const int u = t - 1, su = u & 1;
            if (!wait_bar_all(&sm.p_full[su], (u >> 1) & 1, wc)) break;
            if (!wait_bar_all(&sm.v_full[su], (u >> 1) & 1, wc)) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t b = sdesc_sw128(smem_u32(sm.v[su][0]) + kk * 2048, 64 * 128, 1024);
              mma_ts_el(tmem_o, tmem + su * 64 + kk * 8, b, IDESC_O, (u > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit_el(&sm.v_empty[su]);
            mma_commit_el(&sm.o_done);
          }
        }
      }
      // drain: every MMA issued above completes before TMEM is released
      mma_commit_el(&sm.drain);
      const WaitCtx drain_wc{&sm.never, nullptr, wait_limit_ns};
      wait_bar_all(&sm.drain, 0, drain_wc);
    }
  } else {
    // ---------------- softmax warps 0-3 ----------------
    const int r = threadIdx.x;                       // row in the tile == TMEM lane
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    float m_use = -INFINITY, l = 0.f;
    bool ok = n > 0;
    // only the kv tile Tn-1 is ragged, and the ascending list holds it last
    const int last_valid = (n > 0 && (kv_list[n - 1] & TILE_ID_MASK) == Tn - 1) ? (N - (Tn - 1) * 64) : 64;
    const int half = warp >> 1;  // rows 64*half .. 64*half+63 of the tile
    for (int t = 0; t < n && ok; ++t) {
      const int s = t & 1;
      if (!wait_warp(&sm.s_full[s], (t >> 1) & 1, wc)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // a tile excluded for this row's half (a 64-row query block that does not
      // keep it) contributes nothing: every logit masked
      const bool excl = TILED && tile_excluded(kv_list[t], half);
      const int valid = excl ? 0 : (t == n - 1) ? last_valid : 64;
      uint32_t sv[64];
      tmem_ld64(tl + s * 64, sv);
      tmem_wait_ld();
      if (valid < 64) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c >= valid) sv[c] = __float_as_uint(-INFINITY);
      }
      // row max as a tree (independent partial maxima)
      float m4[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) m4[q] = __uint_as_float(sv[q]);
#pragma unroll
      for (int c = 8; c < 64; ++c) m4[c & 7] = fmaxf(m4[c & 7], __uint_as_float(sv[c]));
      const float mx = fmaxf(fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])),
                             fmaxf(fmaxf(m4[4], m4[5]), fmaxf(m4[6], m4[7])));
      const float m_new = fmaxf(m_use, mx * scale_log2);
      float alpha = 1.f;
      bool rescale = false;
      if (m_use == -INFINITY) {
        m_use = m_new;
      } else if (m_new > m_use + 8.0f) {
        alpha = fast_exp2(m_use - m_new);
        m_use = m_new;
        l *= alpha;
        rescale = true;
      }
      const float neg_m = m_use == -INFINITY ? 0.f : -m_use;  // nothing seen yet: every P is 0
      uint32_t pk[32];
      float rsum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float p0 = fast_exp2(fmaf(__uint_as_float(sv[2 * c]), scale_log2, neg_m));
        const float p1 = fast_exp2(fmaf(__uint_as_float(sv[2 * c + 1]), scale_log2, neg_m));
        rsum[c & 3] += p0 + p1;
        pk[c] = pack_f16(p0, p1);
      }
      const float rs = (rsum[0] + rsum[1]) + (rsum[2] + rsum[3]);
      l += rs;
      tmem_st32(tl + s * 64, pk);
      if (t >= 1 && !wait_warp(&sm.o_done, (t - 1) & 1, wc)) {
        ok = false;
        break;
      }
      if (__any_sync(0xffffffff, rescale)) {
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t ov[32];
          tmem_ld32(tl + 128 + cc * 32, ov);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
          tmem_st32(tl + 128 + cc * 32, ov);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full[s]);
    }
    tmem_wait_st();
    // agree on the epilogue among the 128 softmax threads
    named_bar_sync(1, 128);
    if (threadIdx.x == 0) sm.epi_ok = (n > 0 && !sm.abort_flag) ? 1 : 0;
    named_bar_sync(1, 128);
    ok = sm.epi_ok != 0;
    if (ok) ok = wait_warp(&sm.o_done, (n - 1) & 1, wc);
    ok = __all_sync(0xffffffff, ok);
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t ov[32];
        tmem_ld32(tl + 128 + cc * 32, ov);
        tmem_wait_ld();
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float a = __uint_as_float(ov[2 * c]) * inv_l, b = __uint_as_float(ov[2 * c + 1]) * inv_l;
          hi[c] = pack_bf16(a, b);
          const float2 hf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hi[c]));
          lo[c] = pack_bf16(a - hf.x, b - hf.y);
        }
        const uint32_t u0 = (cc & 1) * 4;
        uint8_t* chunk = sm.q[cc >> 1];
        uint8_t* chunk_lo = &sm.k[0][0][0] + (cc >> 1) * (128 * 128);  // K/V ring is free now
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          *reinterpret_cast<uint4*>(chunk + sw128_offset(r, u0 + e)) =
              make_uint4(hi[4 * e], hi[4 * e + 1], hi[4 * e + 2], hi[4 * e + 3]);
          if (has_olo)
            *reinterpret_cast<uint4*>(chunk_lo + sw128_offset(r, u0 + e)) =
                make_uint4(lo[4 * e], lo[4 * e + 1], lo[4 * e + 2], lo[4 * e + 3]);
        }
      }
      const long long row = (long long)i * 128 + r;
      if (row < N) lse[(long long)bh * N + row] = (m_use + log2f(l)) * 0.69314718055994530942f;
    }
    fence_proxy_async_smem();
    named_bar_sync(1, 128);
    if (threadIdx.x == 0 && sm.epi_ok) {
      for (int c = 0; c < CH; ++c) tma_store_3d(&tm_o, sm.q[c], c * 64, i * 128, bh);
      if (has_olo)
        for (int c = 0; c < CH; ++c) tma_store_3d(&tm_olo, &sm.k[0][0][0] + c * (128 * 128), c * 64, i * 128, bh);
      tma_store_commit();
      tma_store_wait_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// bf16 -> fp16 copy of V; |v| > 65504 is clamped to the largest finite fp16 and
// reported as SPA2_ERR_RANGE. Each thread converts V16_UNROLL 16-byte units a
// block-width apart, all of its loads issued before the first conversion, so a
// thread keeps 64 bytes in flight (one unit at a time left the copy at ~0.8 of
// HBM bandwidth).
constexpr int V16_UNROLL = 4;
__global__ void __launch_bounds__(256) v_to_f16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                       long long n8, int* status) {
  pdl_trigger();  // the forward kernel may start its prologue (Q load, TMEM, barriers)
  bool bad = false;
  const long long base = (long long)blockIdx.x * (256 * V16_UNROLL) + threadIdx.x;
  uint4 v[V16_UNROLL];
#pragma unroll
  for (int u = 0; u < V16_UNROLL; ++u) {
    const long long e = base + u * 256;
    v[u] = e < n8 ? src[e] : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int u = 0; u < V16_UNROLL; ++u) {
    const long long e = base + u * 256;
    const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
      if (!(fabsf(f.x) <= 65504.f) || !(fabsf(f.y) <= 65504.f)) {
        bad = true;
        f.x = fminf(fmaxf(f.x, -65504.f), 65504.f);
        f.y = fminf(fmaxf(f.y, -65504.f), 65504.f);
      }
      o[i] = pack_f16(f.x, f.y);
    }
    if (e < n8) dst[e] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (bad) report(status, SPA2_ERR_RANGE);
}

cudaError_t launch_v_to_f16(const void* v, void* v16, long long elems, int* status, cudaStream_t s) {
  const long long n8 = elems / 8;
  const long long per_block = 256LL * V16_UNROLL;
  const long long blocks = (n8 + per_block - 1) / per_block;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  KernelTimer kt(KID_V16, s);
  return launch_k(v_to_f16_kernel, dim3((unsigned)std::max(blocks, 1LL)), dim3(256), 0, s, false,
                  static_cast<const uint4*>(v), static_cast<uint4*>(v16), n8, status);
}

template <int D, bool TILED>
static cudaError_t launch_fwd_t(const FwdArgs& a, cudaStream_t s) {
  const size_t smem = sizeof(FwdSmem<D>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(fwd_kernel<D, TILED>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_k(fwd_kernel<D, TILED>, dim3(a.Tm, a.BH), dim3(192), smem, s, true, *a.tm_q, *a.tm_k, *a.tm_v,
                  *a.tm_o, *a.tm_olo, a.has_olo, a.row_cnt, a.row_idx, a.lse, a.N, a.Tm, a.Tn, a.scale_log2, a.status,
                  a.wait_limit_ns);
}

cudaError_t launch_fwd(const FwdArgs& a, int d, cudaStream_t s) {
  KernelTimer kt(KID_FWD, s);
  if (d == 128) return a.tiled ? launch_fwd_t<128, true>(a, s) : launch_fwd_t<128, false>(a, s);
  return a.tiled ? launch_fwd_t<64, true>(a, s) : launch_fwd_t<64, false>(a, s);
}

}  // namespace spa2
