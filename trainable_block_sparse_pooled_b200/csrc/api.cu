// C ABI of libspa2 (declared in include/spa2.h): argument validation,
// workspace layout, TMA descriptor construction and kernel launches. No entry
// point allocates device memory; every buffer, the workspace included, belongs
// to the caller.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace spa2 {

static unsigned long long g_wait_limit_ns = 2000000000ull;  // 2 s

static inline size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

struct Shape {
  int B, H, N, d, Tm, Tn, W;
  long long BH;
  int bq, bkv;
  int TMt, TNt;  // 128-row query tiles and 64-row key tiles of the attention kernels
  bool tiled;    // block sizes other than (128, 64): the block lists are converted to tile lists
};

static bool shape_ok(int B, int H, int N, int d, int bq, int bkv, Shape* s, spa2_status* err) {
  if (B < 1 || H < 1 || N < 1) {
    *err = SPA2_ERR_INVALID_ARG;
    return false;
  }
  if ((d != 64 && d != 128) || (bq != 64 && bq != 128 && bq != 256) || (bkv != 64 && bkv != 128) || N > 131072 ||
      (long long)B * H > 65535) {
    *err = SPA2_ERR_UNSUPPORTED;
    return false;
  }
  s->B = B;
  s->H = H;
  s->N = N;
  s->d = d;
  s->BH = (long long)B * H;
  s->Tm = (N + bq - 1) / bq;
  s->Tn = (N + bkv - 1) / bkv;
  s->W = (s->Tn + 31) / 32;
  s->bq = bq;
  s->bkv = bkv;
  s->TMt = (N + 127) / 128;
  s->TNt = (N + 63) / 64;
  s->tiled = bq != 128 || bkv != 64;
  return true;
}

static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static bool frac_ok(float x) { return x >= 0.f && x <= 1.f; }  // false for NaN

// workspace layout -----------------------------------------------------------
struct MaskWs {
  int* status;
  float* qbar;  // Qbar in 64-row chunks [BH, kbar_chunks(Tm), d, 64]
  float* kbc;   // Kbar in 64-key chunks [BH, kbar_chunks(Tn), d, 64]
  float* lg;    // pooled logits [BH, Tm, Tn]
  uint32_t* bits;
  size_t bytes;
};
static MaskWs mask_ws(void* ws, const Shape& s) {
  MaskWs w{};
  size_t off = 256;
  char* base = static_cast<char*>(ws);
  w.status = reinterpret_cast<int*>(base);
  w.qbar = reinterpret_cast<float*>(base + off);
  off += al256((size_t)s.BH * kbar_chunks(s.Tm) * s.d * 64 * 4);
  w.kbc = reinterpret_cast<float*>(base + off);
  off += al256((size_t)s.BH * kbar_chunks(s.Tn) * s.d * 64 * 4);
  w.lg = reinterpret_cast<float*>(base + off);
  off += al256((size_t)s.BH * s.Tm * s.Tn * 4);
  w.bits = reinterpret_cast<uint32_t*>(base + off);
  off += al256((size_t)s.BH * s.Tm * s.W * 4);
  w.bytes = off;
  return w;
}

// tile lists (tiled shapes only): CSR [BH, TMt] counts + [BH, TMt, TNt] entries,
// CSC [BH, TNt] counts + [BH, TNt, TMt] entries
struct TileWs {
  int* csr_cnt;
  int* csr_idx;
  int* csc_cnt;
  int* csc_idx;
};
static size_t tile_ws(char* base, size_t off, const Shape& s, bool csc, TileWs* t) {
  if (!s.tiled) return off;
  t->csr_cnt = reinterpret_cast<int*>(base + off);
  off += al256((size_t)s.BH * s.TMt * 4);
  t->csr_idx = reinterpret_cast<int*>(base + off);
  off += al256((size_t)s.BH * s.TMt * s.TNt * 4);
  if (csc) {
    t->csc_cnt = reinterpret_cast<int*>(base + off);
    off += al256((size_t)s.BH * s.TNt * 4);
    t->csc_idx = reinterpret_cast<int*>(base + off);
    off += al256((size_t)s.BH * s.TNt * s.TMt * 4);
  }
  return off;
}

struct FwdWs {
  int* status;
  void* v16;  // fp16 copy of V [BH, N, d]
  TileWs tiles;
  size_t bytes;
};
static FwdWs fwd_ws(void* ws, const Shape& s) {
  FwdWs w{};
  char* base = static_cast<char*>(ws);
  size_t off = 256;
  w.status = reinterpret_cast<int*>(base);
  w.v16 = base + off;
  off += al256((size_t)s.BH * s.N * s.d * 2);
  w.bytes = tile_ws(base, off, s, false, &w.tiles);
  return w;
}

struct BwdWs {
  int* status;
  float* dvec;
  void* do16;
  void* q16;
  int* col_order;  // the order of the dK/dV pass's columns
  TileWs tiles;
  size_t bytes;
};
static BwdWs bwd_ws(void* ws, const Shape& s) {
  BwdWs w{};
  char* base = static_cast<char*>(ws);
  size_t off = 256;
  w.status = reinterpret_cast<int*>(base);
  w.dvec = reinterpret_cast<float*>(base + off);
  off += al256((size_t)s.BH * s.N * 4);
  w.do16 = base + off;
  off += al256((size_t)s.BH * s.N * s.d * 2);
  w.q16 = base + off;
  off += al256((size_t)s.BH * s.N * s.d * 2);
  w.col_order = reinterpret_cast<int*>(base + off);
  off += al256((size_t)s.BH * s.TNt * 4);
  w.bytes = tile_ws(base, off, s, true, &w.tiles);
  return w;
}

// TMA descriptors ------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

enum MapType { MAP_BF16 = 0, MAP_F16 = 1, MAP_F32 = 2 };

// Descriptor cache: a tensor map depends only on (address, shape, element
// type, box rows), so the maps of buffers reused from call to call are encoded
// once. Small, fixed size, round-robin replacement; guarded by a mutex.
struct MapKey {
  const void* ptr;
  long long BH;
  int N, d, rows, type;
  bool operator==(const MapKey& o) const {
    return ptr == o.ptr && BH == o.BH && N == o.N && d == o.d && rows == o.rows && type == o.type;
  }
};
static constexpr int kMapCache = 64;
static MapKey g_map_key[kMapCache];
static CUtensorMap g_map_val[kMapCache];
static bool g_map_used[kMapCache];
static int g_map_next = 0;
static std::mutex g_map_mu;

// [BH, N, d] viewed as a 3-D tensor {d, N, BH}; box {64 bf16/fp16 or 32 fp32
// columns (128 bytes), rows, 1}, 128-byte swizzle; rows past N of a head read
// as zero (no spill into the next head) and are clipped on stores.
static bool encode_map(CUtensorMap* m, const void* ptr, const Shape& s, int rows, int type) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t esz = type == MAP_F32 ? 4 : 2;
  cuuint64_t dims[3] = {(cuuint64_t)s.d, (cuuint64_t)s.N, (cuuint64_t)s.BH};
  cuuint64_t strides[2] = {(cuuint64_t)s.d * esz, (cuuint64_t)s.N * s.d * esz};
  cuuint32_t box[3] = {type == MAP_F32 ? 32u : 64u, (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType dt = type == MAP_F32   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : type == MAP_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                   : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = fn(m, dt, 3, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static bool get_map(CUtensorMap* m, const void* ptr, const Shape& s, int rows, int type) {
  const MapKey key{ptr, s.BH, s.N, s.d, rows, type};
  std::lock_guard<std::mutex> lock(g_map_mu);
  for (int i = 0; i < kMapCache; ++i)
    if (g_map_used[i] && g_map_key[i] == key) {
      *m = g_map_val[i];
      return true;
    }
  if (!encode_map(m, ptr, s, rows, type)) return false;
  const int slot = g_map_next;
  g_map_next = (g_map_next + 1) % kMapCache;
  g_map_key[slot] = key;
  g_map_val[slot] = *m;
  g_map_used[slot] = true;
  return true;
}

static bool make_map(CUtensorMap* m, const void* ptr, const Shape& s, int rows, bool f16 = false) {
  return get_map(m, ptr, s, rows, f16 ? MAP_F16 : MAP_BF16);
}

static bool make_map_f32(CUtensorMap* m, const void* ptr, const Shape& s, int rows) {
  return get_map(m, ptr, s, rows, MAP_F32);
}

static int topk_count(float k_frac, int Tn) {
  long long K = (long long)floor((double)k_frac * (double)Tn + 0.5);
  if (K < 1) K = 1;
  if (K > Tn) K = Tn;
  return (int)K;
}

static unsigned long long topp_threshold(float p_frac) {
  return (unsigned long long)floor((double)p_frac * 4294967296.0);
}

// device-side timeout probe ----------------------------------------------------
__global__ void timeout_probe_kernel(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const WaitCtx w{&abort_flag, status, limit_ns};
  wait_bar(&bar, 0, w);  // nothing ever arrives: runs out after limit_ns
}

cudaError_t launch_timeout_probe(int* status, unsigned long long limit_ns, cudaStream_t s) {
  KernelTimer kt(KID_PROBE, s);
  timeout_probe_kernel<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace spa2

using namespace spa2;

#define SPA2_CUDA_TRY(expr)                      \
  do {                                           \
    if ((expr) != cudaSuccess) return SPA2_ERR_CUDA; \
  } while (0)

extern "C" {

int spa2_abi_version(void) { return SPA2_ABI_VERSION; }

const char* spa2_status_string(spa2_status s) {
  switch (s) {
    case SPA2_OK: return "ok";
    case SPA2_ERR_INVALID_ARG: return "invalid argument";
    case SPA2_ERR_UNSUPPORTED: return "unsupported shape or parameter";
    case SPA2_ERR_CUDA: return "CUDA call failed";
    case SPA2_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case SPA2_ERR_WORKSPACE: return "workspace missing or too small";
    case SPA2_ERR_DEVICE_BOUNDS: return "device-side index check failed";
    case SPA2_ERR_RANGE: return "input value outside the supported range";
  }
  return "unknown status";
}

size_t spa2_workspace_bytes(int op, int B, int H, int N, int d, int bq, int bkv) {
  Shape s;
  spa2_status err;
  if (op == SPA2_OP_SELECT) {
    if (B < 1 || H < 1 || N < 1 || d < 1) return 0;
    const long long BH = (long long)B * H;
    const long long W = (d + 31) / 32;
    return 256 + al256((size_t)(BH * N * W * 4));
  }
  if (!shape_ok(B, H, N, d, bq, bkv, &s, &err)) return 0;
  switch (op) {
    case SPA2_OP_MASK: return mask_ws(nullptr, s).bytes;
    case SPA2_OP_FWD: return fwd_ws(nullptr, s).bytes;  // status + fp16 V (+ tile lists)
    case SPA2_OP_BWD: return bwd_ws(nullptr, s).bytes;
  }
  return 0;
}

spa2_status spa2_block_mask(const void* q, const void* k, int B, int H, int N, int d, int bq, int bkv, float k_frac,
                            float p_frac, const spa2_mask* out, void* ws, size_t ws_bytes, spa2_stream_t stream) {
  Shape s;
  spa2_status err;
  if (!q || !k || !out || !out->row_cnt || !out->row_idx) return SPA2_ERR_INVALID_ARG;
  if ((out->col_cnt == nullptr) != (out->col_idx == nullptr)) return SPA2_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(out->row_cnt, 4) || !aligned(out->row_idx, 4))
    return SPA2_ERR_INVALID_ARG;
  if (!shape_ok(B, H, N, d, bq, bkv, &s, &err)) return err;
  if (!frac_ok(k_frac) || !frac_ok(p_frac)) return SPA2_ERR_UNSUPPORTED;
  if (!ws || !aligned(ws, 256)) return SPA2_ERR_WORKSPACE;
  MaskWs w = mask_ws(ws, s);
  if (ws_bytes < w.bytes) return SPA2_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  SPA2_CUDA_TRY(cudaMemsetAsync(w.status, 0, 4, st));
  MaskOut mo{out->row_cnt, out->row_idx, out->pbar, out->bitmap};
  SPA2_CUDA_TRY(launch_mask(q, k, w.qbar, w.kbc, w.lg, (int)s.BH, s.N, s.d, s.Tm, s.Tn, bq, bkv, topk_count(k_frac, s.Tn),
                            topp_threshold(p_frac), mo, out->col_cnt, out->col_idx, w.bits, s.W, w.status,
                            g_wait_limit_ns, st));
  return SPA2_OK;
}

spa2_status spa2_select_blocks(const float* pbar, int B, int H, int Tm, int Tn, float k_frac, float p_frac,
                               const spa2_mask* out, void* ws, size_t ws_bytes, spa2_stream_t stream) {
  if (!pbar || !out || !out->row_cnt || !out->row_idx) return SPA2_ERR_INVALID_ARG;
  if ((out->col_cnt == nullptr) != (out->col_idx == nullptr)) return SPA2_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || Tm < 1 || Tn < 1) return SPA2_ERR_INVALID_ARG;
  if (Tn > 2048 || Tm > 65535 || (long long)B * H > 65535) return SPA2_ERR_UNSUPPORTED;
  if (!frac_ok(k_frac) || !frac_ok(p_frac)) return SPA2_ERR_UNSUPPORTED;
  if (!ws || !aligned(ws, 256)) return SPA2_ERR_WORKSPACE;
  const size_t need = spa2_workspace_bytes(SPA2_OP_SELECT, B, H, Tm, Tn, 0, 0);
  if (ws_bytes < need) return SPA2_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  uint32_t* bits = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + 256);
  const int BH = B * H, W = (Tn + 31) / 32;
  SPA2_CUDA_TRY(cudaMemsetAsync(status, 0, 4, st));
  MaskOut mo{out->row_cnt, out->row_idx, nullptr, out->bitmap};
  SPA2_CUDA_TRY(launch_select(pbar, BH, Tm, Tn, topk_count(k_frac, Tn), topp_threshold(p_frac), mo, bits, W, status,
                              st));
  if (out->col_cnt) SPA2_CUDA_TRY(launch_csc(bits, BH, Tm, Tn, W, out->col_cnt, out->col_idx, st));
  return SPA2_OK;
}

spa2_status spa2_sparse_attn_fwd(const void* q, const void* k, const void* v, int B, int H, int N, int d, int bq,
                                 int bkv, const spa2_mask* mask, float softmax_scale, void* o, void* o_lo, float* lse,
                                 void* ws, size_t ws_bytes, spa2_stream_t stream) {
  Shape s;
  spa2_status err;
  if (!q || !k || !v || !o || !lse || !mask || !mask->row_cnt || !mask->row_idx) return SPA2_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(o_lo, 16) ||
      !aligned(lse, 4))
    return SPA2_ERR_INVALID_ARG;
  if (!shape_ok(B, H, N, d, bq, bkv, &s, &err)) return err;
  if (!(softmax_scale >= 0.f) || isinf(softmax_scale)) return SPA2_ERR_UNSUPPORTED;
  if (!ws || !aligned(ws, 256)) return SPA2_ERR_WORKSPACE;
  FwdWs w = fwd_ws(ws, s);
  if (ws_bytes < w.bytes) return SPA2_ERR_WORKSPACE;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)d);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  CUtensorMap tq, tk, tv, to, tolo;
  if (!make_map(&tq, q, s, 128) || !make_map(&tk, k, s, 64) || !make_map(&tv, w.v16, s, 64, true) ||
      !make_map(&to, o, s, 128) || !make_map(&tolo, o_lo ? o_lo : o, s, 128))
    return SPA2_ERR_CUDA;
  int* status = w.status;
  SPA2_CUDA_TRY(cudaMemsetAsync(status, 0, 4, st));
  const int* rc = mask->row_cnt;
  const int* ri = mask->row_idx;
  if (s.tiled) {
    SPA2_CUDA_TRY(launch_tile_lists(mask->row_cnt, mask->row_idx, nullptr, nullptr, (int)s.BH, s.Tm, s.Tn, s.TMt,
                                    s.TNt, s.bq, s.bkv, w.tiles.csr_cnt, w.tiles.csr_idx, nullptr, nullptr, status,
                                    st));
    rc = w.tiles.csr_cnt;
    ri = w.tiles.csr_idx;
  }
  SPA2_CUDA_TRY(launch_v_to_f16(v, w.v16, s.BH * s.N * s.d, status, st));
  FwdArgs a{&tq, &tk, &tv, &to, &tolo, o_lo != nullptr, rc, ri, lse, (int)s.BH, s.N, s.TMt, s.TNt,
            scale * 1.4426950408889634f, status, g_wait_limit_ns, s.tiled ? 1 : 0};
  SPA2_CUDA_TRY(launch_fwd(a, d, st));
  return SPA2_OK;
}

spa2_status spa2_sparse_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* o_lo,
                                 const float* lse, const void* dout, int B, int H, int N, int d, int bq, int bkv,
                                 const spa2_mask* mask, float softmax_scale, void* dq, void* dk, void* dv,
                                 int grad_dtype, void* ws, size_t ws_bytes, spa2_stream_t stream) {
  Shape s;
  spa2_status err;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !mask || !mask->row_cnt || !mask->row_idx ||
      !mask->col_cnt || !mask->col_idx)
    return SPA2_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(o_lo, 16) ||
      !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4))
    return SPA2_ERR_INVALID_ARG;
  if (grad_dtype != SPA2_DTYPE_BF16 && grad_dtype != SPA2_DTYPE_F32) return SPA2_ERR_UNSUPPORTED;
  if (!shape_ok(B, H, N, d, bq, bkv, &s, &err)) return err;
  if (!(softmax_scale >= 0.f) || isinf(softmax_scale)) return SPA2_ERR_UNSUPPORTED;
  if (!ws || !aligned(ws, 256)) return SPA2_ERR_WORKSPACE;
  BwdWs w = bwd_ws(ws, s);
  if (ws_bytes < w.bytes) return SPA2_ERR_WORKSPACE;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)d);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool f32 = grad_dtype == SPA2_DTYPE_F32;
  CUtensorMap tq, tk, tv, tdo, tq16, tdq;
  if (!make_map(&tq, q, s, 128) || !make_map(&tk, k, s, 64) || !make_map(&tv, v, s, 64) ||
      !make_map(&tdo, w.do16, s, 128, true) || !make_map(&tq16, w.q16, s, 128, true) ||
      !(f32 ? make_map_f32(&tdq, dq, s, 128) : make_map(&tdq, dq, s, 128)))
    return SPA2_ERR_CUDA;
  SPA2_CUDA_TRY(cudaMemsetAsync(w.status, 0, 256, st));  // status word and the dK/dV column ticket
  const int *rc = mask->row_cnt, *ri = mask->row_idx, *cc = mask->col_cnt, *ci = mask->col_idx;
  if (s.tiled) {
    SPA2_CUDA_TRY(launch_tile_lists(mask->row_cnt, mask->row_idx, mask->col_cnt, mask->col_idx, (int)s.BH, s.Tm, s.Tn,
                                    s.TMt, s.TNt, s.bq, s.bkv, w.tiles.csr_cnt, w.tiles.csr_idx, w.tiles.csc_cnt,
                                    w.tiles.csc_idx, w.status, st));
    rc = w.tiles.csr_cnt;
    ri = w.tiles.csr_idx;
    cc = w.tiles.csc_cnt;
    ci = w.tiles.csc_idx;
  }
  BwdArgs a{&tq, &tk, &tv, &tdo, &tq16, &tdq, q, k, o, o_lo, dout, v, lse, rc, ri, cc, ci, w.dvec, w.do16,
            w.q16, dq, dk, dv, f32 ? 1 : 0, (int)s.BH, s.N, s.TMt, s.TNt, scale,
            scale * 1.4426950408889634f, w.status, w.status + 32, g_wait_limit_ns, s.tiled ? 1 : 0,
            w.col_order};
  SPA2_CUDA_TRY(launch_bwd(a, d, st));
  return SPA2_OK;
}

spa2_status spa2_stream_status(void* ws, spa2_stream_t stream) {
  if (!ws) return SPA2_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return SPA2_ERR_CUDA;
  int code = 0;
  if (cudaMemcpy(&code, ws, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return SPA2_ERR_CUDA;
  if (cudaMemset(ws, 0, 4) != cudaSuccess) return SPA2_ERR_CUDA;
  return static_cast<spa2_status>(code);
}

spa2_status spa2_debug_set_wait_limit_ns(long long limit) {
  g_wait_limit_ns = limit > 0 ? (unsigned long long)limit : 2000000000ull;
  return SPA2_OK;
}

spa2_status spa2_debug_timeout_probe(void* ws, size_t ws_bytes, spa2_stream_t stream) {
  if (!ws || ws_bytes < 256 || !aligned(ws, 256)) return SPA2_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  SPA2_CUDA_TRY(cudaMemsetAsync(ws, 0, 4, st));
  SPA2_CUDA_TRY(launch_timeout_probe(static_cast<int*>(ws), g_wait_limit_ns, st));
  return SPA2_OK;
}

}  // extern "C"
