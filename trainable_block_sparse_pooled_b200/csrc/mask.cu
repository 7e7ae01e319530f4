// Block-mask kernels: steps 1-3 of SpargeAttention2 (paper.rainbus.top summary,
// 方法步骤详情 steps 1-3; 技术新颖性 union formula; gist.science 2A).
//
//   pool_kernel    one CTA per block, every streaming load of a thread in flight
//                  before it sums: means of the q-blocks and kv-blocks -> Qbar
//                  and Kbar in chunks of 64 blocks, each chunk d x 64
//                  ([B*H, ceil(T_m / 64), d, 64], [B*H, ceil(T_n / 64), d, 64],
//                  fp32).
//   logits_kernel  S-bar = Qbar Kbar^T / sqrt(d), fp32: one CTA per 64 x 64 tile
//                  of one head, both chunks by bulk copy into shared memory,
//                  thread = 4 rows x 4 keys with paired fp32 FMAs -> logit
//                  scratch [B*H, T_m, T_n].
//   select_kernel  one warp per row, the row in registers: softmax -> P-bar,
//                  hybrid selection -> CSR, kept-bit words, optional P-bar /
//                  uint8 bitmap.
//   csc_kernel     kept-bit words -> CSC: one CTA per (head, 32-column word),
//                  32x32 bit transposes with warp ballots.
//   pbar_select_kernel  the selection alone on a caller-given P-bar.
// The four mask kernels run back to back on one stream; each after the first is
// launched as a programmatic dependent of the one before.
//
// Selection is exact integer work on the float32 P-bar: ranks are (value desc,
// id asc); Top-k keeps the first K ranks; Top-p keeps rank r while the
// quantised mass floor(2^32 P) of ranks before r is below floor(2^32 p). Both
// are prefixes of the same order, so the union is the first n = max(K, R)
// ranks, and the value at rank n-1 is the largest key T with
//   count(key >= T) >= K  and  mass(key >= T) >= thr,
// found by one bisection over the float bit patterns (monotone for P >= 0),
// with ties at T taken by ascending block id. No sort, no atomics. Rows that
// keep at most 64 blocks are instead walked rank by rank (extract_top), the
// warp taking the largest key of per-lane top-4 caches at each step. The
// bisection passes over the whole row only until at most 32 keys remain
// between its bounds; those are compacted to one per lane and the rest of the
// search counts them with ballots (keys above the bracket are carried as a
// count and a mass, keys below it never count). Each lane
// keeps its E = ceil(T_n / 32) keys and masses in registers; masses are split
// as q >> 16 and q & 0xffff so warp sums stay exact in 32 bits
// (__reduce_add_sync) for rows of fewer than 2^15 blocks.
#include "common.cuh"
#include "kernels.h"

namespace spa2 {

namespace {

constexpr int ROWS = 8;  // P-bar rows per select CTA (one warp each)

SPA2_DEV unsigned long long mass_of(float p) {
  return __float2ull_rz(p * 4294967296.0f);  // exact: power-of-two scale of p in [0, 1]
}

// ---------------------------------------------------------------------------
// exact hybrid selection of one row by one warp; lane l holds elements l + 32 e,
// e < E, of the row: key = float bits of P-bar (0 for padding), mh / ml = mass
// halves (0 for padding)
// ---------------------------------------------------------------------------
// Kept ids of a row from its kept-bit words (bal[e] bit l = element 32 e + l):
// CSR row in ascending order, kept-bit words, optional uint8 bitmap; checks the
// count against n.
template <int E>
SPA2_DEV void emit_row(const uint32_t (&bal)[E], int Tn, int n, int* row_cnt_out, int* row_idx_out,
                       uint32_t* bits_out, uint8_t* bitmap_out, int* status) {
  const uint32_t lane = lane_id();
  const uint32_t lt = (1u << lane) - 1u;
  int running = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int j = 32 * e + (int)lane;
    if (32 * e < Tn) {
      const bool keep = (bal[e] >> lane) & 1u;
      if (keep) row_idx_out[running + __popc(bal[e] & lt)] = j;
      if (bitmap_out && j < Tn) bitmap_out[j] = keep ? 1 : 0;
      if (lane == 0) bits_out[e] = bal[e];
      running += __popc(bal[e]);
    }
  }
  if (lane == 0) {
    *row_cnt_out = running;
    if (running != n) report(status, SPA2_ERR_DEVICE_BOUNDS);
  }
}

// Exact rank-order walk for rows that keep few blocks. Ranks are taken one at a
// time as the warp maximum of (key desc, id asc): every lane keeps its own
// best 4 not-yet-taken elements in a sorted cache of packed 64-bit values
// (refilled from its registers when it runs dry), the warp takes the largest cached key (REDUX max) and,
// among lanes holding that key, the lowest block id (REDUX min). Rank r is kept
// while r < K or the mass of ranks < r is below thr, exactly the rule of the
// bisection below. Returns false, having changed nothing, when the row keeps
// more than EXTRACT_CAP ranks; otherwise kept = this lane's kept elements (bit
// e = element lane + 32 e) and n = their count over the warp.
constexpr int EXTRACT_CAP = 64;

// This lane's best 4 elements not yet taken, as packed 64-bit values
// ((key + 1) << 8 | (255 - e)): a larger value is a higher rank (larger key,
// then smaller e); 0 marks an empty slot. Kept sorted, hk[0] the best.
template <int E>
SPA2_DEV void top4_refill(const uint32_t (&key)[E], int Tn, uint64_t taken, uint64_t (&hk)[4]) {
  const uint32_t lane = lane_id();
#pragma unroll
  for (int j = 0; j < 4; ++j) hk[j] = 0ull;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    uint64_t v = ((int)lane + 32 * e < Tn && !((taken >> e) & 1ull))
                     ? ((uint64_t)(key[e] + 1u) << 8) | (uint64_t)(255 - e)
                     : 0ull;
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // insertion by compare-exchange
      const uint64_t hi = v > hk[j] ? v : hk[j];
      v = v > hk[j] ? hk[j] : v;
      hk[j] = hi;
    }
  }
}

template <int E>
SPA2_DEV bool extract_top(const uint32_t (&key)[E], int Tn, int K, unsigned long long thr, uint64_t& kept,
                          int& n_out) {
  const uint32_t lane = lane_id();
  uint64_t hk[4];
  kept = 0ull;
  top4_refill<E>(key, Tn, kept, hk);
  int mine = 0;  // valid elements of this lane not yet taken
#pragma unroll
  for (int e = 0; e < E; ++e) mine += ((int)lane + 32 * e < Tn) ? 1 : 0;
  unsigned long long before = 0ull;  // mass of the ranks taken so far
  for (int r = 0; r <= EXTRACT_CAP; ++r) {
    if (r == Tn) {  // every block taken
      n_out = r;
      return true;
    }
    if (hk[0] == 0ull && mine > 0) top4_refill<E>(key, Tn, kept, hk);
    const uint32_t hkey = (uint32_t)(hk[0] >> 8);  // key + 1, or 0
    const uint32_t gmax = __reduce_max_sync(0xffffffff, hkey);
    const uint32_t id = (hkey == gmax) ? lane + 32u * (255u - (uint32_t)(hk[0] & 255u)) : 0xFFFFFFFFu;
    const uint32_t wid = __reduce_min_sync(0xffffffff, id);
    if (!(r < K || before < thr)) {  // rank r is the first one dropped
      n_out = r;
      return true;
    }
    if (r == EXTRACT_CAP) break;
    before += mass_of(__uint_as_float(gmax - 1u));
    if (lane == (wid & 31u)) {
      kept |= 1ull << (wid >> 5);
      --mine;
      hk[0] = hk[1];
      hk[1] = hk[2];
      hk[2] = hk[3];
      hk[3] = 0ull;
    }
  }
  kept = 0ull;
  return false;
}

template <int E>
SPA2_DEV uint32_t eq_all_ties(const uint32_t (&key)[E], uint32_t bv, int Tn) {
  uint32_t eq = 0u;
#pragma unroll
  for (int e = 0; e < E; ++e) eq += ((int)lane_id() + 32 * e < Tn && key[e] == bv) ? 1u : 0u;
  return __reduce_add_sync(0xffffffff, eq);
}

template <int E>
SPA2_DEV void select_row_regs(const uint32_t (&key)[E], int Tn, int K, unsigned long long thr, int* row_cnt_out,
                              int* row_idx_out, uint32_t* bits_out, uint8_t* bitmap_out, int* status,
                              uint32_t* scratch /* 96 words, this warp's */) {
  const uint32_t lane = lane_id();
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t bal[E];
  if (K < Tn && K <= EXTRACT_CAP) {
    uint64_t kept;
    int n_kept;
    if (extract_top<E>(key, Tn, K, thr, kept, n_kept)) {
#pragma unroll
      for (int e = 0; e < E; ++e) bal[e] = __ballot_sync(0xffffffff, (kept >> e) & 1ull);
      emit_row<E>(bal, Tn, n_kept, row_cnt_out, row_idx_out, bits_out, bitmap_out, status);
      return;
    }
  }
  // bisection path: quantised masses, split into 16-bit halves
  uint32_t mh[E], ml[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const unsigned long long q = mass_of(__uint_as_float(key[e]));  // padding keys are 0: mass 0
    mh[e] = (uint32_t)(q >> 16);
    ml[e] = (uint32_t)(q & 0xffffull);
  }
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
    // Every mid tested is > lo >= 0, so padding keys (0) never count. cnt_lo /
    // cnt_hi are the numbers of valid keys >= lo / >= hi, m_hi the mass of the
    // keys >= hi; keys in [lo, hi) are the only ones the remaining tests can split.
    uint32_t lo = kmin, hi = kmax + 1u;
    uint32_t cnt_lo = (uint32_t)Tn, cnt_hi = 0u;
    unsigned long long m_hi = 0ull;
    // phase A: passes over the whole row until at most 32 keys lie in [lo, hi)
#pragma unroll 1
    while (hi - lo > 1u && cnt_lo - cnt_hi > 32u) {
      const uint32_t mid = lo + ((hi - lo) >> 1);
      uint32_t c = 0u, sh = 0u, sl = 0u;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const bool in = key[e] >= mid;
        c += in ? 1u : 0u;
        sh += in ? mh[e] : 0u;
        sl += in ? ml[e] : 0u;
      }
      c = __reduce_add_sync(0xffffffff, c);
      const unsigned long long mass =
          ((unsigned long long)__reduce_add_sync(0xffffffff, sh) << 16) + __reduce_add_sync(0xffffffff, sl);
      if (c >= (uint32_t)K && mass >= thr) {
        lo = mid;
        cnt_lo = c;
      } else {
        hi = mid;
        cnt_hi = c;
        m_hi = mass;
      }
    }
    // phase B: the <= 32 keys in [lo, hi) compacted to one per lane; keys >= hi
    // enter through cnt_hi / m_hi, keys < lo never count
    if (hi - lo > 1u) {
      uint32_t base = 0u;
      const uint32_t below = (1u << lane) - 1u;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const bool cand = ((int)lane + 32 * e < Tn) && key[e] >= lo && key[e] < hi;
        const uint32_t bal = __ballot_sync(0xffffffff, cand);
        if (cand) {
          const uint32_t pos = base + __popc(bal & below);
          scratch[pos] = key[e];
          scratch[32 + pos] = mh[e];
          scratch[64 + pos] = ml[e];
        }
        base += __popc(bal);
      }
      __syncwarp();
      // Each lane counts the candidates >= its own key (itself and ties included):
      // count(key >= own) = cnt_hi + that, and likewise the mass. The largest
      // candidate key meeting both bounds is the answer; with none, lo is.
      const bool have = lane < base;
      const uint32_t own = have ? scratch[lane] : 0u;
      uint32_t cge = 0u, sh = 0u, sl = 0u;
#pragma unroll 4
      for (uint32_t t = 0; t < base; ++t) {
        const bool ge = scratch[t] >= own;
        cge += ge ? 1u : 0u;
        sh += ge ? scratch[32 + t] : 0u;
        sl += ge ? scratch[64 + t] : 0u;
      }
      __syncwarp();
      const unsigned long long mass = m_hi + ((unsigned long long)sh << 16) + sl;
      const bool meets = have && cnt_hi + cge >= (uint32_t)K && mass >= thr;
      lo = max(lo, __reduce_max_sync(0xffffffff, meets ? own : 0u));
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
      // ceil((thr - gm) / qv) ties, at most eq: a double quotient (both operands
      // < 2^34, so it is within one of the exact one) corrected in integers
      const unsigned long long qv = mass_of(__uint_as_float(lo));  // > 0: mass(key >= T) > mass(key > T)
      const unsigned long long rem = thr - gm;
      unsigned long long need = (unsigned long long)ceil((double)rem / (double)qv);
      if (need > 0ull && (need - 1ull) * qv >= rem) --need;
      if (need * qv < rem) ++need;
      tR = (uint32_t)(need < (unsigned long long)eq ? need : (unsigned long long)eq);
    }
    bv = lo;
    bt = max(tK, tR);
    n = (int)(gt + bt);
    keep_all = (n >= Tn);
  }
  // emit ascending ids: key > bv, or key == bv among the first bt by id
  if (keep_all || bt == 0u || bt >= eq_all_ties(key, bv, Tn)) {
    // no tie needs ranking: every tie at bv is kept (bt >= their count) or none is
    const bool ties_in = !keep_all && bt != 0u;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const bool valid = (int)lane + 32 * e < Tn;
      bal[e] = __ballot_sync(0xffffffff, valid && (keep_all || key[e] > bv || (ties_in && key[e] == bv)));
    }
  } else {
    uint32_t ties_seen = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const bool valid = (int)lane + 32 * e < Tn;
      const bool is_tie = valid && (key[e] == bv);
      const uint32_t tie_bal = __ballot_sync(0xffffffff, is_tie);
      const uint32_t tie_rank = ties_seen + __popc(tie_bal & lt);
      bal[e] = __ballot_sync(0xffffffff, valid && (key[e] > bv || (is_tie && tie_rank < bt)));
      ties_seen += __popc(tie_bal);
    }
  }
  emit_row<E>(bal, Tn, n, row_cnt_out, row_idx_out, bits_out, bitmap_out, status);
}

// load a P-bar row (smem or global, length Tn) into lane registers and select
template <int E>
SPA2_DEV void select_row(const float* row, int Tn, int K, unsigned long long thr, int* row_cnt_out,
                         int* row_idx_out, uint32_t* bits_out, uint8_t* bitmap_out, int* status, uint32_t* scratch) {
  uint32_t key[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int j = (int)lane_id() + 32 * e;
    key[e] = __float_as_uint(j < Tn ? row[j] : 0.f);
  }
  select_row_regs<E>(key, Tn, K, thr, row_cnt_out, row_idx_out, bits_out, bitmap_out, status, scratch);
}


// softmax of one logit row (length Tn, already scaled by 1/sqrt(d)) and its
// selection, by one warp with the row in lane registers: P = exp2((x - max)
// log2 e) / sum, the sum inverted once; P-bar written to pbar_out when it is
// not NULL
template <int E>
SPA2_DEV void softmax_select_row(const float* __restrict__ lrow, int Tn, int K, unsigned long long thr,
                                 float* pbar_out, int* row_cnt_out, int* row_idx_out, uint32_t* bits_out,
                                 uint8_t* bitmap_out, int* status, uint32_t* scratch) {
  constexpr float LOG2E = 1.4426950408889634f;
  const int lane = (int)lane_id();
  float x[E];
  float mx = -INFINITY;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int j = lane + 32 * e;
    x[e] = j < Tn ? lrow[j] : -INFINITY;
  }
#pragma unroll
  for (int e = 0; e < E; ++e) mx = fmaxf(mx, x[e]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffff, mx, o));
  const float nm = -mx * LOG2E;
  float ssum = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    x[e] = fast_exp2(fmaf(x[e], LOG2E, nm));  // 0 for padding (exp2(-inf))
    ssum += x[e];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ssum += __shfl_xor_sync(0xffffffff, ssum, o);
  const float inv = 1.0f / ssum;
  uint32_t key[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int j = lane + 32 * e;
    const float p = j < Tn ? x[e] * inv : 0.f;
    if (pbar_out && j < Tn) pbar_out[j] = p;
    key[e] = __float_as_uint(p);
  }
  select_row_regs<E>(key, Tn, K, thr, row_cnt_out, row_idx_out, bits_out, bitmap_out, status, scratch);
}

// CSC of 32 kv-block columns (one kept-bit word w of every row) of one head:
// for each tile of 32 q-block rows a warp transposes the 32x32 bit block with
// ballots (lane b then holds the bits of column 32w+b over the tile's rows),
// counts are scanned across the tiles in shared memory, and every lane writes
// the ascending row ids of its column.
SPA2_DEV void csc_word_cta(const uint32_t* __restrict__ head_bits, int Tm, int Tn, int W, int w,
                           int* __restrict__ col_cnt, int* __restrict__ col_idx, int* cnt_smem /* [8][32] */,
                           int* base_smem /* [32] */) {
  const int warp = threadIdx.x >> 5;
  const int lane = (int)lane_id();
  const int col = w * 32 + lane;
  if (threadIdx.x < 32) base_smem[lane] = 0;
  __syncthreads();
  for (int t0 = 0; t0 < Tm; t0 += 8 * 32) {  // 8 row tiles of 32 per pass, one per warp
    const int r0 = t0 + warp * 32;
    const int row = r0 + lane;
    const uint32_t word = row < Tm ? head_bits[(long long)row * W + w] : 0u;
    uint32_t mine = 0u;
#pragma unroll
    for (int b = 0; b < 32; ++b) {
      const uint32_t v = __ballot_sync(0xffffffffu, (word >> b) & 1u);
      if (lane == b) mine = v;
    }
    cnt_smem[warp * 32 + lane] = __popc(mine);
    __syncthreads();
    int pos = base_smem[lane];
    for (int u = 0; u < warp; ++u) pos += cnt_smem[u * 32 + lane];
    if (col < Tn) {
      int* dst = col_idx + (long long)col * Tm + pos;
      while (mine) {
        const int bit = __ffs(mine) - 1;
        mine &= mine - 1u;
        *dst++ = r0 + bit;
      }
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      int tot = 0;
      for (int u = 0; u < 8; ++u) tot += cnt_smem[u * 32 + lane];
      base_smem[lane] += tot;
    }
    __syncthreads();
  }
  if (threadIdx.x < 32 && col < Tn) col_cnt[col] = base_smem[lane];
}

}  // namespace

constexpr int LG_C = 64;  // rows (keys) per Qbar (Kbar) chunk: one logits tile is 64 x 64

// Pooling: one CTA of 256 threads per block (blockIdx.x < T_m: q-block ->
// Qbar; otherwise kv-block -> Kbar chunk column). Each thread owns a
// 16-byte column chunk of every 16th (d = 128) or 32nd (d = 64) row and issues
// all of its streaming loads of a 128-row span before summing; partial sums
// meet in shared memory.
template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                   const __nv_bfloat16* __restrict__ k, float* __restrict__ qbar,
                                                   float* __restrict__ kbc, int N, int Tm, int Tn, int bq,
                                                   int bkv) {
  constexpr int TPR = D / 8;        // threads per row (8 bf16 each)
  constexpr int RP = 256 / TPR;     // rows per pass
  constexpr int MAXIT = 128 / RP;   // loads per thread per 128-row span
  __shared__ float red[RP * (D + 1)];
  pdl_trigger();  // the select kernel may be scheduled; it waits for this grid before reading
  const int blk = blockIdx.x;
  const long long h = blockIdx.y;
  const bool is_q = blk < Tm;
  const int idx = is_q ? blk : blk - Tm;
  const int bsz = is_q ? bq : bkv;
  const int rows = min(bsz, N - idx * bsz);
  const __nv_bfloat16* src = (is_q ? q : k) + (h * N + (long long)idx * bsz) * D;
  const int tr = threadIdx.x / TPR, tc = threadIdx.x % TPR;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  const uint4* base = reinterpret_cast<const uint4*>(src) + tc;
  for (int r0 = 0; r0 < rows; r0 += 128) {
    uint4 v[MAXIT];
#pragma unroll
    for (int u = 0; u < MAXIT; ++u) {
      const int r = r0 + tr + u * RP;
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
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[tr * (D + 1) + tc * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float sum = 0.f;
#pragma unroll 8
    for (int i = 0; i < RP; ++i) sum += red[i * (D + 1) + threadIdx.x];
    const float mean = sum / static_cast<float>(rows);
    if (is_q)
      qbar[((h * ((Tm + LG_C - 1) / LG_C) + (idx >> 6)) * D + threadIdx.x) * LG_C + (idx & 63)] = mean;
    else
      kbc[((h * ((Tn + LG_C - 1) / LG_C) + (idx >> 6)) * D + threadIdx.x) * LG_C + (idx & 63)] = mean;
  }
}

// Pooled logits: S-bar = Qbar Kbar^T / sqrt(d) -> lg [B*H, Tm, Tn] fp32. CTA
// (key chunk, row chunk, head) of 128 threads computes one 64 x 64 tile: both
// chunks (d x 64 each) arrive by bulk copy; thread (ty, tx) holds rows
// 8ty..8ty+7 x keys 4tx..4tx+3 and adds, for d in order, two 16-byte loads of
// its rows (four row pairs) and one of its keys: four key-pair registers and
// sixteen paired fp32 FMAs (two products each) per column, the loads of four
// columns issued ahead of their FMAs; then scales by 1/sqrt(d).
template <int D>
struct LogitSmem {
  static constexpr int CHUNK_BYTES = D * LG_C * 4;
  static constexpr int TOTAL = 2 * CHUNK_BYTES;  // Kbar chunk, then Qbar chunk
};

template <int D>
__global__ void __launch_bounds__(128, 3) logits_kernel(const float* __restrict__ qbar, const float* __restrict__ kbc,
                                                     float* __restrict__ lg, int Tm, int Tn, float inv_sqrt_d,
                                                     int* status, unsigned long long wait_limit_ns) {
  using L = LogitSmem<D>;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  const float* ks = reinterpret_cast<const float*>(smem);
  const float* qs = reinterpret_cast<const float*>(smem + L::CHUNK_BYTES);
  const int c = blockIdx.x, C = gridDim.x, rq = blockIdx.y, CQ = gridDim.y;
  const long long h = blockIdx.z;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();     // Qbar and Kbar are complete
  pdl_trigger();  // the select kernel may be scheduled; it waits for this grid itself
  if (threadIdx.x == 0) {
    mbar_expect_tx(&bar, 2u * L::CHUNK_BYTES);
    bulk_load(smem, kbc + (h * C + c) * D * LG_C, L::CHUNK_BYTES, &bar);
    bulk_load(smem + L::CHUNK_BYTES, qbar + (h * CQ + rq) * D * LG_C, L::CHUNK_BYTES, &bar);
  }
  const WaitCtx wc{&abort_flag, status, wait_limit_ns};
  wait_bar(&bar, 0, wc);
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  uint64_t acc[4][4];  // [row pair][key]: {row 8ty + 2p, row 8ty + 2p + 1}
#pragma unroll
  for (int p = 0; p < 4; ++p)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[p][j] = 0ull;
  const ulonglong2* qrow = reinterpret_cast<const ulonglong2*>(qs) + 2 * ty;  // column dd at qrow[dd * 16], +1
  const float4* kcol = reinterpret_cast<const float4*>(ks) + tx;              // column dd at kcol[dd * 16]
#pragma unroll 1
  for (int d0 = 0; d0 < D; d0 += 4) {
    ulonglong2 qa[4], qb[4];
    float4 kv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      qa[u] = qrow[(d0 + u) * (LG_C / 4)];
      qb[u] = qrow[(d0 + u) * (LG_C / 4) + 1];
      kv[u] = kcol[(d0 + u) * (LG_C / 4)];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint64_t kk[4] = {f2_pack(kv[u].x, kv[u].x), f2_pack(kv[u].y, kv[u].y), f2_pack(kv[u].z, kv[u].z),
                              f2_pack(kv[u].w, kv[u].w)};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc[0][j] = f2_fma(qa[u].x, kk[j], acc[0][j]);
        acc[1][j] = f2_fma(qa[u].y, kk[j], acc[1][j]);
        acc[2][j] = f2_fma(qb[u].x, kk[j], acc[2][j]);
        acc[3][j] = f2_fma(qb[u].y, kk[j], acc[3][j]);
      }
    }
  }
  const int j0 = c * LG_C + 4 * tx;
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    float lo[4], hi[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) f2_unpack(acc[p][j], lo[j], hi[j]);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int r = rq * LG_C + 8 * ty + 2 * p + u;
      if (r >= Tm) continue;
      float* dst = lg + (h * Tm + r) * Tn + j0;
      const float* v = u ? hi : lo;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (j0 + j < Tn) dst[j] = v[j] * inv_sqrt_d;
    }
  }
}

// Softmax and selection, one warp per P-bar row (4 rows per CTA): the row's
// logits from lg, P-bar in registers, CSR, kept-bit words, optional P-bar /
// uint8 bitmap.
template <int E>
__global__ void __launch_bounds__(128, (E <= 16 ? 6 : 2)) select_kernel(const float* __restrict__ lg, long long R,
                                                                       int Tn, int W, int K, unsigned long long thr,
                                                                       MaskOut out, uint32_t* __restrict__ bits,
                                                                       int* status) {
  __shared__ uint32_t scr[4][96];
  pdl_wait();     // the logits are complete
  pdl_trigger();  // the CSC kernel may be scheduled; it waits for this grid itself
  const int warp = (int)(threadIdx.x >> 5);
  const long long rowid = (long long)blockIdx.x * 4 + warp;
  if (rowid >= R) return;
  softmax_select_row<E>(lg + rowid * Tn, Tn, K, thr, out.pbar ? out.pbar + rowid * Tn : nullptr, out.row_cnt + rowid,
                        out.row_idx + rowid * Tn, bits + rowid * W, out.bitmap ? out.bitmap + rowid * Tn : nullptr,
                        status, scr[warp]);
}

// selection alone on a given P-bar: one warp per row, 8 rows per CTA
template <int E>
__global__ void __launch_bounds__(256) pbar_select_kernel(const float* __restrict__ pbar, int Tm, int Tn, int W,
                                                          int K, unsigned long long thr, MaskOut out,
                                                          uint32_t* __restrict__ bits, int* status) {
  pdl_trigger();
  const int w = threadIdx.x >> 5;
  const long long bh = blockIdx.y;
  const int i = blockIdx.x * 8 + w;
  if (i >= Tm) return;
  __shared__ uint32_t scr[8][96];
  const long long rowid = bh * Tm + i;
  select_row<E>(pbar + rowid * Tn, Tn, K, thr, out.row_cnt + rowid, out.row_idx + rowid * Tn, bits + rowid * W,
                out.bitmap ? out.bitmap + rowid * Tn : nullptr, status, scr[w]);
}

// kept-bit words [B*H, Tm, W] -> CSC; one CTA per (32-column word, head)
__global__ void __launch_bounds__(256) csc_kernel(const uint32_t* __restrict__ bits, int Tm, int Tn, int W,
                                                  int* __restrict__ col_cnt, int* __restrict__ col_idx) {
  __shared__ int cnt_smem[8 * 32];
  __shared__ int base_smem[32];
  pdl_wait();  // the kept-bit words are complete
  const long long bh = blockIdx.y;
  csc_word_cta(bits + bh * Tm * W, Tm, Tn, W, blockIdx.x, col_cnt + bh * Tn, col_idx + bh * Tn * Tm, cnt_smem,
               base_smem);
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
int kbar_chunks(int Tn) { return (Tn + LG_C - 1) / LG_C; }

template <int E>
static cudaError_t launch_select_t(const float* lg, int BH, int Tm, int Tn, int W, int K, unsigned long long thr,
                                   const MaskOut& out, uint32_t* bits, int* status, cudaStream_t s) {
  const long long R = (long long)BH * Tm;
  KernelTimer kt(KID_SELECT, s);
  return launch_k(select_kernel<E>, dim3((unsigned)((R + 3) / 4)), dim3(128), 0, s, true, lg, R, Tn, W, K, thr, out,
                  bits, status);
}

static cudaError_t launch_select_e(const float* lg, int BH, int Tm, int Tn, int W, int K, unsigned long long thr,
                                   const MaskOut& out, uint32_t* bits, int* status, cudaStream_t s) {
  const int e = (Tn + 31) / 32;
  if (e <= 8) return launch_select_t<8>(lg, BH, Tm, Tn, W, K, thr, out, bits, status, s);
  if (e <= 16) return launch_select_t<16>(lg, BH, Tm, Tn, W, K, thr, out, bits, status, s);
  if (e <= 40) return launch_select_t<40>(lg, BH, Tm, Tn, W, K, thr, out, bits, status, s);
  return launch_select_t<64>(lg, BH, Tm, Tn, W, K, thr, out, bits, status, s);
}

template <int D>
static cudaError_t launch_logits_d(const float* qbar, const float* kbc, float* lg, int BH, int Tm, int Tn, int* status,
                                   unsigned long long wait_limit_ns, cudaStream_t s) {
  constexpr int kMaxDev = 64;
  static bool attr_set[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 0 || dev >= kMaxDev || !attr_set[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(logits_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               LogitSmem<D>::TOTAL);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDev) attr_set[dev] = true;
  }
  KernelTimer kt(KID_LOGITS, s);
  return launch_k(logits_kernel<D>, dim3(kbar_chunks(Tn), kbar_chunks(Tm), BH), dim3(128),
                  (size_t)LogitSmem<D>::TOTAL, s, true, qbar, kbc, lg, Tm, Tn, 1.0f / sqrtf((float)D), status,
                  wait_limit_ns);
}

template <int D>
static cudaError_t launch_pool_d(const void* q, const void* k, float* qbar, float* kbc, int BH, int N, int Tm, int Tn,
                                 int bq, int bkv, cudaStream_t s) {
  KernelTimer kt(KID_POOL, s);
  return launch_k(pool_kernel<D>, dim3(Tm + Tn, BH), dim3(256), 0, s, false, static_cast<const __nv_bfloat16*>(q),
                  static_cast<const __nv_bfloat16*>(k), qbar, kbc, N, Tm, Tn, bq, bkv);
}

cudaError_t launch_mask(const void* q, const void* k, float* qbar, float* kbc, float* lg, int BH, int N, int d,
                        int Tm, int Tn, int bq, int bkv, int K, unsigned long long thr, const MaskOut& out,
                        int* col_cnt, int* col_idx, uint32_t* bits, int W, int* status,
                        unsigned long long wait_limit_ns, cudaStream_t s) {
  cudaError_t e = d == 128 ? launch_pool_d<128>(q, k, qbar, kbc, BH, N, Tm, Tn, bq, bkv, s)
                           : launch_pool_d<64>(q, k, qbar, kbc, BH, N, Tm, Tn, bq, bkv, s);
  if (e != cudaSuccess) return e;
  e = d == 128 ? launch_logits_d<128>(qbar, kbc, lg, BH, Tm, Tn, status, wait_limit_ns, s)
               : launch_logits_d<64>(qbar, kbc, lg, BH, Tm, Tn, status, wait_limit_ns, s);
  if (e != cudaSuccess) return e;
  e = launch_select_e(lg, BH, Tm, Tn, W, K, thr, out, bits, status, s);
  if (e != cudaSuccess) return e;
  if (col_cnt) {
    KernelTimer kt(KID_CSC, s);
    e = launch_k(csc_kernel, dim3(W, BH), dim3(256), 0, s, true, static_cast<const uint32_t*>(bits), Tm, Tn, W,
                 col_cnt, col_idx);
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
  KernelTimer kt(KID_CSC, s);
  return launch_k(csc_kernel, dim3(W, BH), dim3(256), 0, s, true, bits, Tm, Tn, W, col_cnt, col_idx);
}

}  // namespace spa2
