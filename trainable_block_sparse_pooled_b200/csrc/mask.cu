// Block-mask kernels: steps 1-3 of SpargeAttention2 (paper.rainbus.top summary,
// 方法步骤详情 steps 1-3; 技术新颖性 union formula; gist.science 2A).
//
//   pool_kernel    one CTA per block: mean of each q-block (b_q rows) and kv-block
//                  (b_kv rows) of Q / K -> Qbar [B,H,Tm,d], Kbar [B,H,Tn,d] fp32.
//   select_kernel  8 q-block rows of one head per CTA, one warp per row: fp32
//                  logits against Kbar (streamed through a 4-deep smem ring with
//                  bulk async copies), softmax -> P-bar, hybrid selection -> CSR,
//                  kept-bit words, optional P-bar / uint8 bitmap.
//   csc_kernel     kept-bit words -> CSC, one warp per kv-block column.
//   pbar_select_kernel  the selection alone on a caller-given P-bar.
//
// Selection is exact integer work on the float32 P-bar: ranks are (value desc,
// id asc); Top-k keeps the first K ranks; Top-p keeps rank r while the
// quantised mass floor(2^32 P) of ranks before r is below floor(2^32 p). Both
// are prefixes of the same order, so the union is the first n = max(K, R)
// ranks, and the value at rank n-1 is the largest key T with
//   count(key >= T) >= K  and  mass(key >= T) >= thr,
// found by one bisection over the float bit patterns (monotone for P >= 0),
// with ties at T taken by ascending block id. No sort, no atomics. Each lane
// keeps its E = ceil(T_n / 32) keys and masses in registers; masses are split
// as q >> 16 and q & 0xffff so warp sums stay exact in 32 bits
// (__reduce_add_sync) for rows of fewer than 2^15 blocks.
#include "common.cuh"
#include "kernels.h"

namespace spa2 {

namespace {

constexpr int ROWS = 8;  // P-bar rows per select CTA (one warp each)
constexpr int KCH = 32;  // Kbar rows per staged chunk

SPA2_DEV unsigned long long mass_of(float p) {
  return __float2ull_rz(p * 4294967296.0f);  // exact: power-of-two scale of p in [0, 1]
}

// ---------------------------------------------------------------------------
// pooling of one block: 16-byte streaming loads, all rows of a thread in flight
// ---------------------------------------------------------------------------
template <int D>
SPA2_DEV void pool_block(const __nv_bfloat16* __restrict__ src, int rows, float* __restrict__ dst, float* red) {
  constexpr int TPR = D / 8;     // threads per row (8 bf16 each)
  constexpr int RP = 256 / TPR;  // rows per pass
  constexpr int MAXIT = 128 / RP;
  const int tr = threadIdx.x / TPR, tc = threadIdx.x % TPR;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  const uint4* base = reinterpret_cast<const uint4*>(src) + tc;
  uint4 v[MAXIT];
#pragma unroll
  for (int u = 0; u < MAXIT; ++u) {
    const int r = tr + u * RP;
    v[u] = (r < rows) ? __ldcs(base + (long long)r * TPR) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int u = 0; u < MAXIT; ++u) {
    const __nv_bfloat162* hp = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(hp[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[tr * (D + 1) + tc * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
#pragma unroll 8
    for (int i = 0; i < RP; ++i) s += red[i * (D + 1) + threadIdx.x];
    dst[threadIdx.x] = s / static_cast<float>(rows);
  }
}

// ---------------------------------------------------------------------------
// exact hybrid selection of one row by one warp; lane l holds elements l + 32 e,
// e < E, of the row: key = float bits of P-bar (0 for padding), mh / ml = mass
// halves (0 for padding)
// ---------------------------------------------------------------------------
template <int E>
SPA2_DEV void select_row_regs(const uint32_t (&key)[E], const uint32_t (&mh)[E], const uint32_t (&ml)[E], int Tn,
                              int K, unsigned long long thr, int* row_cnt_out, int* row_idx_out, uint32_t* bits_out,
                              uint8_t* bitmap_out, int* status) {
  const uint32_t lane = lane_id();
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u, th = 0u, tl = 0u;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const bool valid = (int)lane + 32 * e < Tn;
    kmin = valid ? min(kmin, key[e]) : kmin;
    kmax = max(kmax, key[e]);
    th += mh[e];
    tl += ml[e];
  }
  kmin = __reduce_min_sync(0xffffffff, kmin);
  kmax = __reduce_max_sync(0xffffffff, kmax);
  const unsigned long long total =
      ((unsigned long long)__reduce_add_sync(0xffffffff, th) << 16) + __reduce_add_sync(0xffffffff, tl);

  uint32_t bv = 0u, bt = 0u;
  bool keep_all = (K >= Tn) || (thr > total);  // every rank stays below p: Top-p keeps all
  int n = Tn;
  if (!keep_all) {
    // largest T with count(key >= T) >= K and mass(key >= T) >= thr; T = kmin satisfies
    // both (count Tn >= K, mass = total >= thr), T = kmax + 1 satisfies neither
    uint32_t lo = kmin, hi = kmax + 1u;
#pragma unroll 1
    while (hi - lo > 1u) {
      const uint32_t mid = lo + ((hi - lo) >> 1);
      uint32_t c = 0u, sh = 0u, sl = 0u;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const bool in = key[e] >= mid;  // padding keys are 0 < mid
        c += in ? 1u : 0u;
        sh += in ? mh[e] : 0u;
        sl += in ? ml[e] : 0u;
      }
      c = __reduce_add_sync(0xffffffff, c);
      const unsigned long long mass =
          ((unsigned long long)__reduce_add_sync(0xffffffff, sh) << 16) + __reduce_add_sync(0xffffffff, sl);
      if (c >= (uint32_t)K && mass >= thr) lo = mid; else hi = mid;
    }
    uint32_t gt = 0u, eq = 0u, gh = 0u, gl = 0u;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const bool valid = (int)lane + 32 * e < Tn;
      gt += (valid && key[e] > lo) ? 1u : 0u;
      eq += (valid && key[e] == lo) ? 1u : 0u;
      gh += (key[e] > lo) ? mh[e] : 0u;
      gl += (key[e] > lo) ? ml[e] : 0u;
    }
    gt = __reduce_add_sync(0xffffffff, gt);
    eq = __reduce_add_sync(0xffffffff, eq);
    const unsigned long long gm =
        ((unsigned long long)__reduce_add_sync(0xffffffff, gh) << 16) + __reduce_add_sync(0xffffffff, gl);
    // ties Top-k needs at T, and ties the inclusive Top-p walk keeps at T
    const uint32_t tK = ((uint32_t)K > gt) ? (uint32_t)K - gt : 0u;
    uint32_t tR = 0u;
    if (thr > gm) {
      const unsigned long long qv = mass_of(__uint_as_float(lo));  // > 0: mass(key >= T) > mass(key > T)
      const unsigned long long need = (thr - gm + qv - 1ull) / qv;
      tR = (uint32_t)(need < (unsigned long long)eq ? need : (unsigned long long)eq);
    }
    bv = lo;
    bt = max(tK, tR);
    n = (int)(gt + bt);
    keep_all = (n >= Tn);
  }
  // emit ascending ids: key > bv, or key == bv among the first bt by id
  const uint32_t lt = (1u << lane) - 1u;
  int running = 0;
  uint32_t ties_seen = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    if (32 * e >= Tn) break;
    const int j = 32 * e + (int)lane;
    const bool valid = j < Tn;
    const uint32_t u = key[e];
    const bool is_tie = valid && (u == bv);
    const uint32_t tie_bal = __ballot_sync(0xffffffff, is_tie);
    const uint32_t tie_rank = ties_seen + __popc(tie_bal & lt);
    const bool keep = valid && (keep_all || u > bv || (is_tie && tie_rank < bt));
    const uint32_t bal = __ballot_sync(0xffffffff, keep);
    if (keep) row_idx_out[running + __popc(bal & lt)] = j;
    if (bitmap_out && valid) bitmap_out[j] = keep ? 1 : 0;
    if (lane == 0) bits_out[e] = bal;
    running += __popc(bal);
    ties_seen += __popc(tie_bal);
  }
  if (lane == 0) {
    *row_cnt_out = running;
    if (running != n) report(status, SPA2_ERR_DEVICE_BOUNDS);
  }
}

// load a P-bar row (smem or global, length Tn) into lane registers and select
template <int E>
SPA2_DEV void select_row(const float* row, int Tn, int K, unsigned long long thr, int* row_cnt_out,
                         int* row_idx_out, uint32_t* bits_out, uint8_t* bitmap_out, int* status) {
  uint32_t key[E], mh[E], ml[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int j = (int)lane_id() + 32 * e;
    const float p = j < Tn ? row[j] : 0.f;
    const unsigned long long q = mass_of(p);
    key[e] = __float_as_uint(p);
    mh[e] = (uint32_t)(q >> 16);
    ml[e] = (uint32_t)(q & 0xffffull);
  }
  select_row_regs<E>(key, mh, ml, Tn, K, thr, row_cnt_out, row_idx_out, bits_out, bitmap_out, status);
}

// CSC of one kv-block column c by one warp (ascending q-block ids)
SPA2_DEV void csc_column_warp(const uint32_t* __restrict__ head_bits, int Tm, int W, int c, int* col_cnt_out,
                              int* col_idx_out) {
  const uint32_t lane = lane_id();
  const uint32_t lt = (1u << lane) - 1u;
  const uint32_t* col = head_bits + (c >> 5);
  int running = 0;
  for (int base = 0; base < Tm; base += 32 * 8) {
    uint32_t w8[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {  // all loads of 8 row groups in flight
      const int i = base + 32 * u + (int)lane;
      w8[u] = (i < Tm) ? col[(long long)i * W] : 0u;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + 32 * u + (int)lane;
      const bool bit = (w8[u] >> (c & 31)) & 1u;
      const uint32_t bal = __ballot_sync(0xffffffff, bit);
      if (bit) col_idx_out[running + __popc(bal & lt)] = i;
      running += __popc(bal);
    }
  }
  if (lane == 0) *col_cnt_out = running;
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                   const __nv_bfloat16* __restrict__ k, float* __restrict__ qbar,
                                                   float* __restrict__ kbar, int h0, int N, int Tm, int Tn, int bq,
                                                   int bkv) {
  __shared__ float red[(256 / (D / 8)) * (D + 1)];
  const int blk = blockIdx.x;
  const long long h = h0 + blockIdx.y;
  const __nv_bfloat16* src;
  float* dst;
  int rows;
  if (blk < Tm) {
    src = q + (h * N + (long long)blk * bq) * D;
    rows = min(bq, N - blk * bq);
    dst = qbar + (h * Tm + blk) * D;
  } else {
    const int j = blk - Tm;
    src = k + (h * N + (long long)j * bkv) * D;
    rows = min(bkv, N - j * bkv);
    dst = kbar + (h * Tn + j) * D;
  }
  pool_block<D>(src, rows, dst, red);
}

// 8 rows (one per warp) of head h0 + blockIdx.y: logits, softmax, selection
template <int D, int E>
__global__ void __launch_bounds__(256, (E <= 16 ? 2 : 1)) select_kernel(const float* __restrict__ qbar,
                                                        const float* __restrict__ kbar, int h0, int Tm, int Tn, int W,
                                                        float inv_sqrt_d, int K, unsigned long long thr, MaskOut out,
                                                        uint32_t* __restrict__ bits, int* status,
                                                        unsigned long long wait_limit_ns) {
  constexpr int NST = 4;                                   // ring depth
  extern __shared__ __align__(128) unsigned char smem_raw[];
  float* ring = reinterpret_cast<float*>(smem_raw);        // [NST][KCH][D], unpadded
  float* qb = ring + NST * KCH * D;                        // [ROWS][D]
  float* lrows = qb + ROWS * D;                            // [ROWS][32 E]
  uint64_t* full = reinterpret_cast<uint64_t*>(lrows + ROWS * 32 * E);  // [NST]
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5;
  const uint32_t lane = lane_id();
  const long long h = h0 + blockIdx.y;
  const int i0 = blockIdx.x * ROWS;
  const float* kb = kbar + h * Tn * D;
  const int nch = (Tn + KCH - 1) / KCH;
  if (threadIdx.x == 0) {
    for (int st = 0; st < NST; ++st) mbar_init(&full[st], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const WaitCtx wc{&abort_flag, status, wait_limit_ns};
  int issued = 0;  // meaningful in thread 0 only
  auto issue = [&](int ch) {  // thread 0 only
    const int rows = min(KCH, Tn - ch * KCH);
    const uint32_t bytes = (uint32_t)rows * D * 4;
    uint64_t* bar = &full[ch % NST];
    mbar_expect_tx(bar, bytes);
    bulk_load(ring + (ch % NST) * KCH * D, kb + (long long)ch * KCH * D, bytes, bar);
    issued = ch + 1;
  };
  if (threadIdx.x == 0)
    for (int ch = 0; ch < min(NST - 1, nch); ++ch) issue(ch);
  for (int e = threadIdx.x; e < ROWS * D; e += 256) {
    const int rr = e / D;
    qb[e] = (i0 + rr < Tm) ? qbar[(h * Tm + i0 + rr) * D + (e % D)] : 0.f;
  }
  __syncthreads();
  float* lrow = lrows + warp * 32 * E;
  const float4* qr = reinterpret_cast<const float4*>(qb + warp * D);
  bool ok = true;
  int ch = 0;
  for (; ch < nch; ++ch) {
    if (threadIdx.x == 0 && ch + NST - 1 < nch) issue(ch + NST - 1);  // its slot was freed last iteration
    ok = wait_bar(&full[ch % NST], (ch / NST) & 1, wc);
    if (__syncthreads_or(!ok)) {
      ok = false;
      break;
    }
    // lane l: logit of row (i0 + warp) against Kbar row ch*KCH + l; each lane walks
    // d in its own rotated order (conflict-free 16-byte smem reads), sequentially
    const int c = ch * KCH + (int)lane;
    if (c < Tn) {
      const float4* kr = reinterpret_cast<const float4*>(ring + (ch % NST) * KCH * D + lane * D);
      float acc = 0.f;
#pragma unroll 8
      for (int t = 0; t < D / 4; ++t) {
        const int e = (t + (int)lane) & (D / 4 - 1);
        const float4 kv = kr[e];
        const float4 qv = qr[e];
        acc = fmaf(qv.x, kv.x, acc);
        acc = fmaf(qv.y, kv.y, acc);
        acc = fmaf(qv.z, kv.z, acc);
        acc = fmaf(qv.w, kv.w, acc);
      }
      lrow[c] = acc * inv_sqrt_d;
    }
    __syncthreads();  // every warp is done with this slot
  }
  if (!ok) {
    // never leave with bulk copies in flight: wait (bounded) for the issued ones
    if (threadIdx.x == 0) {
      __shared__ int never;
      never = 0;
      const WaitCtx dw{&never, nullptr, wait_limit_ns};
      for (int c2 = ch; c2 < issued; ++c2) wait_bar(&full[c2 % NST], (c2 / NST) & 1, dw);
    }
    return;
  }
  const int i = i0 + warp;
  if (i >= Tm) return;
  float mx = -INFINITY;
  for (int j = lane; j < Tn; j += 32) mx = fmaxf(mx, lrow[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffff, mx, o));
  float ssum = 0.f;
  for (int j = lane; j < Tn; j += 32) {
    const float e = expf(lrow[j] - mx);
    lrow[j] = e;
    ssum += e;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ssum += __shfl_xor_sync(0xffffffff, ssum, o);
  const long long rowid = h * Tm + i;
  for (int j = lane; j < Tn; j += 32) {
    const float p = lrow[j] / ssum;
    lrow[j] = p;
    if (out.pbar) out.pbar[rowid * Tn + j] = p;
  }
  __syncwarp();
  select_row<E>(lrow, Tn, K, thr, out.row_cnt + rowid, out.row_idx + rowid * Tn, bits + rowid * W,
                out.bitmap ? out.bitmap + rowid * Tn : nullptr, status);
}

// selection alone on a given P-bar: one warp per row, 8 rows per CTA
template <int E>
__global__ void __launch_bounds__(256) pbar_select_kernel(const float* __restrict__ pbar, int Tm, int Tn, int W,
                                                          int K, unsigned long long thr, MaskOut out,
                                                          uint32_t* __restrict__ bits, int* status) {
  const int w = threadIdx.x >> 5;
  const long long bh = blockIdx.y;
  const int i = blockIdx.x * 8 + w;
  if (i >= Tm) return;
  const long long rowid = bh * Tm + i;
  select_row<E>(pbar + rowid * Tn, Tn, K, thr, out.row_cnt + rowid, out.row_idx + rowid * Tn, bits + rowid * W,
                out.bitmap ? out.bitmap + rowid * Tn : nullptr, status);
}

// kept-bit words [B*H, Tm, W] -> CSC; one warp per kv-block column, 8 per CTA
__global__ void __launch_bounds__(256) csc_kernel(const uint32_t* __restrict__ bits, int h0, int Tm, int Tn,
                                                  int W, int* __restrict__ col_cnt, int* __restrict__ col_idx) {
  const long long bh = h0 + blockIdx.y;
  const int c = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (c >= Tn) return;
  csc_column_warp(bits + bh * Tm * W, Tm, W, c, col_cnt + bh * Tn + c, col_idx + (bh * Tn + c) * Tm);
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
template <int D, int E>
static cudaError_t launch_select_t(const float* qbar, const float* kbar, int h0, int nh, int Tm, int Tn, int W, int K,
                                   unsigned long long thr, const MaskOut& out, uint32_t* bits, int* status,
                                   unsigned long long wait_limit_ns, cudaStream_t s) {
  const size_t smem = ((size_t)4 * KCH * D + (size_t)ROWS * D + (size_t)ROWS * 32 * E) * 4 + 4 * 8;
  cudaError_t e = cudaFuncSetAttribute(select_kernel<D, E>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  KernelTimer kt(KID_SELECT, s);
  select_kernel<D, E><<<dim3((Tm + ROWS - 1) / ROWS, nh), 256, smem, s>>>(
      qbar, kbar, h0, Tm, Tn, W, 1.0f / sqrtf((float)D), K, thr, out, bits, status, wait_limit_ns);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_select_d(const float* qbar, const float* kbar, int h0, int nh, int Tm, int Tn, int W, int K,
                                   unsigned long long thr, const MaskOut& out, uint32_t* bits, int* status,
                                   unsigned long long wl, cudaStream_t s) {
  const int e = (Tn + 31) / 32;
  if (e <= 8) return launch_select_t<D, 8>(qbar, kbar, h0, nh, Tm, Tn, W, K, thr, out, bits, status, wl, s);
  if (e <= 16) return launch_select_t<D, 16>(qbar, kbar, h0, nh, Tm, Tn, W, K, thr, out, bits, status, wl, s);
  if (e <= 40) return launch_select_t<D, 40>(qbar, kbar, h0, nh, Tm, Tn, W, K, thr, out, bits, status, wl, s);
  return launch_select_t<D, 64>(qbar, kbar, h0, nh, Tm, Tn, W, K, thr, out, bits, status, wl, s);
}

cudaError_t launch_mask(const void* q, const void* k, float* qbar, float* kbar, int BH, int N, int d, int Tm, int Tn,
                        int bq, int bkv, int K, unsigned long long thr, const MaskOut& out, int* col_cnt,
                        int* col_idx, uint32_t* bits, int W, int* status, unsigned long long wait_limit_ns,
                        cudaStream_t s) {
  dim3 grid(Tm + Tn, BH);
  {
  KernelTimer kt(KID_POOL, s);
  if (d == 128)
    pool_kernel<128><<<grid, 256, 0, s>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k, qbar, kbar, 0, N, Tm, Tn,
                                          bq, bkv);
  else
    pool_kernel<64><<<grid, 256, 0, s>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k, qbar, kbar, 0, N, Tm, Tn,
                                         bq, bkv);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = (d == 128) ? launch_select_d<128>(qbar, kbar, 0, BH, Tm, Tn, W, K, thr, out, bits, status, wait_limit_ns, s)
                 : launch_select_d<64>(qbar, kbar, 0, BH, Tm, Tn, W, K, thr, out, bits, status, wait_limit_ns, s);
  if (e != cudaSuccess) return e;
  if (col_cnt) {
    KernelTimer kt(KID_CSC, s);
    csc_kernel<<<dim3((Tn + 7) / 8, BH), 256, 0, s>>>(bits, 0, Tm, Tn, W, col_cnt, col_idx);
    e = cudaGetLastError();
  }
  return e;
}

cudaError_t launch_select(const float* pbar, int BH, int Tm, int Tn, int K, unsigned long long thr,
                          const MaskOut& out, uint32_t* bits, int W, int* status, cudaStream_t s) {
  dim3 grid((Tm + 7) / 8, BH);
  const int e = (Tn + 31) / 32;
  KernelTimer kt(KID_PBAR_SELECT, s);
  if (e <= 8)
    pbar_select_kernel<8><<<grid, 256, 0, s>>>(pbar, Tm, Tn, W, K, thr, out, bits, status);
  else if (e <= 16)
    pbar_select_kernel<16><<<grid, 256, 0, s>>>(pbar, Tm, Tn, W, K, thr, out, bits, status);
  else if (e <= 40)
    pbar_select_kernel<40><<<grid, 256, 0, s>>>(pbar, Tm, Tn, W, K, thr, out, bits, status);
  else
    pbar_select_kernel<64><<<grid, 256, 0, s>>>(pbar, Tm, Tn, W, K, thr, out, bits, status);
  return cudaGetLastError();
}

cudaError_t launch_csc(const uint32_t* bits, int BH, int Tm, int Tn, int W, int* col_cnt, int* col_idx,
                       cudaStream_t s) {
  dim3 grid((Tn + 7) / 8, BH);
  KernelTimer kt(KID_CSC, s);
  csc_kernel<<<grid, 256, 0, s>>>(bits, 0, Tm, Tn, W, col_cnt, col_idx);
  return cudaGetLastError();
}

}  // namespace spa2
