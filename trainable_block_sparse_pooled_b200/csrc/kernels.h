// Internal launcher declarations of libspa2 (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace spa2 {

// timing.cu: per-kernel event timing (spa2_timing_*). One id per kernel kind.
enum KernelId : int {
  KID_POOL = 0,
  KID_SELECT,
  KID_LOGITS,
  KID_CSC,
  KID_PBAR_SELECT,
  KID_V16,
  KID_FWD,
  KID_BWD_PRE,
  KID_BWD_DKDV,
  KID_BWD_DQ,
  KID_PROBE,
  KID_TILES,
  KID_COUNT
};

// Brackets one kernel launch with two CUDA events recorded on `s` while timing
// is on (construct it just before the launch, in the launch's scope).
class KernelTimer {
 public:
  KernelTimer(int kid, cudaStream_t s);
  ~KernelTimer();
  KernelTimer(const KernelTimer&) = delete;
  KernelTimer& operator=(const KernelTimer&) = delete;

 private:
  int slot_;
  cudaStream_t s_;
};

struct MaskOut {
  int* row_cnt;
  int* row_idx;
  float* pbar;       // may be null
  uint8_t* bitmap;   // may be null
};

// mask.cu
// qbar, kbc: Qbar and Kbar workspaces in chunks of 64 blocks,
// [BH, kbar_chunks(Tm), d, 64] and [BH, kbar_chunks(Tn), d, 64] fp32;
// lg: logit workspace [BH, Tm, Tn] fp32
int kbar_chunks(int Tn);
cudaError_t launch_mask(const void* q, const void* k, float* qbar, float* kbc, float* lg, int BH, int N, int d,
                        int Tm, int Tn, int bq, int bkv, int K, unsigned long long thr, const MaskOut& out,
                        int* col_cnt, int* col_idx, uint32_t* bits, int W, int* status,
                        unsigned long long wait_limit_ns, cudaStream_t s);
cudaError_t launch_select(const float* pbar, int BH, int Tm, int Tn, int K, unsigned long long thr,
                          const MaskOut& out, uint32_t* bits, int W, int* status, cudaStream_t s);
cudaError_t launch_csc(const uint32_t* bits, int BH, int Tm, int Tn, int W, int* col_cnt, int* col_idx,
                       cudaStream_t s);

// attn_fwd.cu
struct FwdArgs {
  const CUtensorMap* tm_q;   // box {64, 128, 1}
  const CUtensorMap* tm_k;   // box {64, 64, 1}
  const CUtensorMap* tm_v;   // box {64, 64, 1}, fp16 copy of V
  const CUtensorMap* tm_o;   // box {64, 128, 1}
  const CUtensorMap* tm_olo; // box {64, 128, 1}; O residual, used when has_olo
  int has_olo;
  const int* row_cnt;
  const int* row_idx;
  float* lse;
  int BH, N, Tm, Tn;
  float scale_log2;   // softmax_scale * log2(e)
  int* status;
  unsigned long long wait_limit_ns;
  int tiled;          // list entries may carry tile exclusion bits
};
cudaError_t launch_fwd(const FwdArgs& a, int d, cudaStream_t s);
cudaError_t launch_v_to_f16(const void* v, void* v16, long long elems, int* status, cudaStream_t s);

// attn_bwd.cu
struct BwdArgs {
  const CUtensorMap* tm_q;    // Q bf16, box {64, 128, 1}
  const CUtensorMap* tm_k;    // K bf16, box {64, 64, 1}
  const CUtensorMap* tm_v;    // V bf16, box {64, 64, 1}
  const CUtensorMap* tm_do;   // fp16 copy of dO, box {64, 128, 1}
  const CUtensorMap* tm_q16;  // fp16 copy of Q, box {64, 128, 1}
  const CUtensorMap* tm_dq;   // dQ output: fp32 box {32, 128, 1} or bf16 box {64, 128, 1}, 128-byte swizzle
  const void* q;
  const void* k;
  const void* o;
  const void* o_lo;   // may be null
  const void* dout;
  const void* v;
  const float* lse;
  const int* row_cnt;
  const int* row_idx;
  const int* col_cnt;
  const int* col_idx;
  float* dvec;     // [BH, N]
  void* do16;      // [BH, N, d] fp16
  void* q16;       // [BH, N, d] fp16
  void* dq;
  void* dk;
  void* dv;
  int grad_f32;       // 1: dq/dk/dv are fp32, 0: bf16
  int BH, N, Tm, Tn;
  float scale;        // softmax_scale
  float scale_log2;   // softmax_scale * log2(e)
  int* status;
  int* ticket;        // zero at launch: the persistent dK/dV kernel's column counter
  unsigned long long wait_limit_ns;
  int tiled;          // list entries may carry tile exclusion bits
  int* col_order;     // [BH * Tn]: the dK/dV pass's columns, head by head, long columns first (pre-pass)
};
cudaError_t launch_bwd(const BwdArgs& a, int d, cudaStream_t s);

// api.cu
cudaError_t launch_timeout_probe(int* status, unsigned long long limit_ns, cudaStream_t s);

// tiles.cu: block CSR (and CSC when csc_cnt is not NULL) -> tile lists of 128-row query tiles x 64-row key
// tiles (TMt = ceil(N / 128), TNt = ceil(N / 64)); see the tile-list notes in common.cuh
cudaError_t launch_tile_lists(const int* row_cnt, const int* row_idx, const int* col_cnt, const int* col_idx, int BH,
                              int Tm, int Tn, int TMt, int TNt, int bq, int bkv, int* csr_cnt, int* csr_idx,
                              int* csc_cnt, int* csc_idx, int* status, cudaStream_t s);

}  // namespace spa2
