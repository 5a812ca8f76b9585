// mmsp.cu -- the C ABI of libmmsp.so (declared in include/mmsp.h): host-side
// validation, TMA descriptor encoding and stream-ordered launches of the
// sm_100a kernels. One translation unit so that every kernel shares the
// device-side timeout flag. The library makes no runtime allocation; its
// only device memory of its own is the fixed module-scope scratch of
// mmsp_attn_bwd_noalloc.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <initializer_list>
#include <mutex>

#include "mmsp.h"
#include "ptx.cuh"
#include "shard.cuh"
#include "merge.cuh"
#include "attn_fwd.cuh"
#include "attn_bwd.cuh"
#include "rope.cuh"
#include "ulysses.cuh"

using namespace mmsp;

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int ok() {
  g_err[0] = 0;
  return MMSP_OK;
}

#define MMSP_CUDA(call)                                                                        \
  do {                                                                                         \
    cudaError_t e_ = (call);                                                                   \
    if (e_ != cudaSuccess) return fail(MMSP_ECUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  int sms = 0;
  bool fwd_attr[4] = {false, false, false, false};
  bool bwd_attr[2] = {false, false};
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

int current_device(int* dev) {
  MMSP_CUDA(cudaGetDevice(dev));
  if (*dev < 0 || *dev >= kMaxDevices) return fail(MMSP_EUNSUPPORTED, "device index %d out of range", *dev);
  return MMSP_OK;
}

int device_sms(int dev, int* sms) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_dev[dev].sms == 0) {
    int v = 0;
    MMSP_CUDA(cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev));
    g_dev[dev].sms = v;
  }
  *sms = g_dev[dev].sms;
  return MMSP_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int get_encode() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode) return MMSP_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || fn == nullptr || q != cudaDriverEntryPointSuccess)
    return fail(MMSP_ECUDA, "cuTensorMapEncodeTiled entry point unavailable");
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return MMSP_OK;
}

// [rows][H][D] bf16 viewed as 3-D (d, head, row); boxes of 64 d x 1 head x
// 128 rows with 128-byte swizzle (one 128-byte line per row and box).
int tmap_rows_heads(CUtensorMap* m, const void* ptr, int64_t rows, int H, int D) {
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MMSP_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MMSP_OK;
}

// Caps for the device-side bounded waits, in SM clock cycles (about 2 s).
constexpr long long kWaitCapCycles = 1LL << 32;

int check_common(int64_t N, int32_t P) {
  if (N < 0) return fail(MMSP_EINVAL, "N must be >= 0 (got %lld)", (long long)N);
  if (P < 1) return fail(MMSP_EINVAL, "P must be >= 1 (got %d)", P);
  if (N >= (int64_t(1) << 31)) return fail(MMSP_EINVAL, "N must be < 2^31 (got %lld)", (long long)N);
  if (N % (2 * (int64_t)P) != 0) return fail(MMSP_EINVAL, "N (%lld) must be divisible by 2P (%d)", (long long)N, 2 * P);
  return MMSP_OK;
}

int check_ranks(int32_t P, int32_t rank_begin, int32_t rank_end) {
  if (rank_begin < 0 || rank_end <= rank_begin || rank_end > P)
    return fail(MMSP_EINVAL, "need 0 <= rank_begin < rank_end <= P (got %d, %d, P=%d)", rank_begin, rank_end, P);
  return MMSP_OK;
}

int check_heads(int32_t Hq, int32_t Hkv, int32_t d) {
  if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return fail(MMSP_EINVAL, "need Hq %% Hkv == 0, Hq, Hkv >= 1 (Hq=%d Hkv=%d)", Hq, Hkv);
  if (d != 64 && d != 128) return fail(MMSP_EINVAL, "head dim d must be 64 or 128 (got %d)", d);
  return MMSP_OK;
}

}  // namespace

extern "C" {

const char* mmsp_last_error(void) { return g_err; }

const char* mmsp_version(void) { return "mmsp 0.1 (sm_100a)"; }

int mmsp_shard(const int32_t* seg_len, const uint8_t* seg_kind, int32_t n_seg, int64_t N, int32_t P,
               int32_t* local2global, int32_t* global2local, uint8_t* modality_local, int32_t* segid_local,
               int32_t* rank_counts, const void* src, void* dst, int64_t row_bytes, int32_t inverse, void* stream) {
  int rc = check_common(N, P);
  if (rc) return rc;
  const bool need_seg = modality_local || segid_local || rank_counts;
  if (need_seg) {
    if (!seg_len || !seg_kind) return fail(MMSP_EINVAL, "segment table required for modality/segid/rank_counts");
    if (n_seg < 1 || n_seg > MMSP_MAX_SEGMENTS)
      return fail(MMSP_EINVAL, "n_seg must be in [1, %d] (got %d)", MMSP_MAX_SEGMENTS, n_seg);
  }
  if ((src == nullptr) != (dst == nullptr)) return fail(MMSP_EINVAL, "src and dst must both be set or both NULL");
  if (src) {
    if (row_bytes <= 0 || row_bytes % 4) return fail(MMSP_EINVAL, "row_bytes must be a positive multiple of 4");
    const uintptr_t al = (row_bytes % 16 == 0) ? 15u : 3u;
    if (((uintptr_t)src | (uintptr_t)dst) & al)
      return fail(MMSP_EINVAL, "src/dst must be %d-byte aligned for row_bytes %lld", (int)al + 1, (long long)row_bytes);
    const char* s = static_cast<const char*>(src);
    const char* e = static_cast<const char*>(dst);
    const int64_t bytes = N * row_bytes;
    if (s < e + bytes && e < s + bytes) return fail(MMSP_EINVAL, "src and dst overlap");
  }
  static SegTable tab;  // host staging; copied into the launch parameters
  static std::mutex tab_mu;
  std::lock_guard<std::mutex> lk(tab_mu);
  if (need_seg) {
    int64_t acc = 0;
    tab.n = n_seg;
    for (int i = 0; i < n_seg; ++i) {
      if (seg_len[i] < 1) return fail(MMSP_EINVAL, "segment %d has length %d < 1", i, seg_len[i]);
      if (seg_kind[i] > 1) return fail(MMSP_EINVAL, "segment %d has kind %d (0 text, 1 visual)", i, seg_kind[i]);
      tab.start[i] = (int32_t)acc;
      tab.kind[i] = seg_kind[i];
      acc += seg_len[i];
      if (acc > N) break;
    }
    if (acc != N) return fail(MMSP_EINVAL, "segment lengths sum to %lld, expected N=%lld", (long long)acc, (long long)N);
    tab.start[n_seg] = (int32_t)N;
  } else {
    tab.n = 0;
    tab.start[0] = 0;
  }
  if (N == 0) return ok();
  int dev, sms;
  if ((rc = current_device(&dev)) || (rc = device_sms(dev, &sms))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (local2global || global2local || modality_local || segid_local) {
    // two blocks per SM: every block first copies the segment starts from
    // the parameter space into shared memory, so more blocks mostly add
    // copies (measured at N = 512K: 8.8 us at 2 per SM, 13.4 us at 8)
    int64_t blocks = (N + 255) / 256;
    if (blocks > 2LL * sms) blocks = 2LL * sms;
    shard_maps_kernel<<<(unsigned)blocks, 256, 0, st>>>(tab, (int32_t)N, P, local2global, global2local,
                                                         modality_local, segid_local);
    MMSP_CUDA(cudaGetLastError());
  }
  if (rank_counts) {
    shard_counts_kernel<<<1, 256, 0, st>>>(tab, (int32_t)N, P, rank_counts);
    MMSP_CUDA(cudaGetLastError());
  }
  if (src) {
    int64_t blocks = (N + 7) / 8;  // 8 warps (rows) per block
    if (blocks > 16LL * sms) blocks = 16LL * sms;
    if (row_bytes % 16 == 0)
      shard_rows_kernel<<<(unsigned)blocks, 256, 0, st>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst),
                                                           (int32_t)N, P, row_bytes / 16, inverse ? 1 : 0);
    else
      shard_rows_words_kernel<<<(unsigned)blocks, 256, 0, st>>>(static_cast<const uint32_t*>(src),
                                                                 static_cast<uint32_t*>(dst), (int32_t)N, P,
                                                                 row_bytes / 4, inverse ? 1 : 0);
    MMSP_CUDA(cudaGetLastError());
  }
  return ok();
}

int mmsp_doc_starts(const int32_t* doc_len, int32_t n_doc, int64_t N, int32_t* doc_start, void* stream) {
  if (N < 0 || N > INT32_MAX) return fail(MMSP_EINVAL, "N must be in [0, 2^31-1]");
  if (!doc_len || !doc_start) return fail(MMSP_EINVAL, "doc_len and doc_start must be non-NULL");
  if ((uintptr_t)doc_start & 3u) return fail(MMSP_EINVAL, "doc_start must be 4-byte aligned");
  if (N == 0) return ok();
  if (n_doc < 1 || n_doc > MMSP_MAX_SEGMENTS)
    return fail(MMSP_EINVAL, "n_doc must be in [1, %d] (got %d)", MMSP_MAX_SEGMENTS, n_doc);
  static SegTable tab;
  static std::mutex tab_mu;
  std::lock_guard<std::mutex> lk(tab_mu);
  int64_t acc = 0;
  tab.n = n_doc;
  for (int i = 0; i < n_doc; ++i) {
    if (doc_len[i] < 1) return fail(MMSP_EINVAL, "document %d has length %d < 1", i, doc_len[i]);
    tab.start[i] = (int32_t)acc;
    tab.kind[i] = 0;
    acc += doc_len[i];
    if (acc > N) break;
  }
  if (acc != N) return fail(MMSP_EINVAL, "document lengths sum to %lld, expected N=%lld", (long long)acc, (long long)N);
  tab.start[n_doc] = (int32_t)N;
  int dev, sms, rc;
  if ((rc = current_device(&dev)) || (rc = device_sms(dev, &sms))) return rc;
  int64_t blocks = (N + 255) / 256;
  if (blocks > 8LL * sms) blocks = 8LL * sms;
  doc_starts_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(tab, (int32_t)N, doc_start);
  MMSP_CUDA(cudaGetLastError());
  return ok();
}

int mmsp_shard_frames(const int32_t* seg_len, const uint8_t* seg_kind, int32_t n_seg, int64_t N, int32_t P,
                      int32_t* global2enc, int32_t* local2enc, int32_t* enc_counts, void* stream) {
  int rc = check_common(N, P);
  if (rc) return rc;
  if (!seg_len || !seg_kind) return fail(MMSP_EINVAL, "seg_len and seg_kind must be non-NULL");
  if (N > 0 && (n_seg < 1 || n_seg > MMSP_MAX_SEGMENTS))
    return fail(MMSP_EINVAL, "n_seg must be in [1, %d] (got %d)", MMSP_MAX_SEGMENTS, n_seg);
  if (((uintptr_t)global2enc | (uintptr_t)local2enc | (uintptr_t)enc_counts) & 3u)
    return fail(MMSP_EINVAL, "outputs must be 4-byte aligned");
  if (N == 0) return ok();
  static SegTable tab;
  static std::mutex tab_mu;
  std::lock_guard<std::mutex> lk(tab_mu);
  int64_t acc = 0;
  tab.n = n_seg;
  for (int i = 0; i < n_seg; ++i) {
    if (seg_len[i] < 1) return fail(MMSP_EINVAL, "segment %d has length %d < 1", i, seg_len[i]);
    if (seg_kind[i] > 1) return fail(MMSP_EINVAL, "segment %d has kind %d (0 text, 1 visual)", i, seg_kind[i]);
    tab.start[i] = (int32_t)acc;
    tab.kind[i] = seg_kind[i];
    acc += seg_len[i];
    if (acc > N) break;
  }
  if (acc != N) return fail(MMSP_EINVAL, "segment lengths sum to %lld, expected N=%lld", (long long)acc, (long long)N);
  tab.start[n_seg] = (int32_t)N;
  if (!global2enc && !local2enc && !enc_counts) return ok();
  int dev, sms;
  if ((rc = current_device(&dev)) || (rc = device_sms(dev, &sms))) return rc;
  int64_t blocks = (N + 255) / 256;
  if (blocks > 8LL * sms) blocks = 8LL * sms;
  frame_maps_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(tab, (int32_t)N, P, global2enc,
                                                                                      local2enc, enc_counts);
  MMSP_CUDA(cudaGetLastError());
  return ok();
}

int mmsp_gather_rows(const void* src, void* dst, const int32_t* index, int64_t n_rows, int64_t row_bytes,
                     int32_t scatter, void* stream) {
  if (n_rows < 0 || n_rows >= (int64_t(1) << 31)) return fail(MMSP_EINVAL, "n_rows must be in [0, 2^31)");
  if (row_bytes <= 0 || row_bytes % 16) return fail(MMSP_EINVAL, "row_bytes must be a positive multiple of 16");
  if (scatter != 0 && scatter != 1) return fail(MMSP_EINVAL, "scatter must be 0 or 1");
  if (n_rows == 0) return ok();
  if (!src || !dst || !index) return fail(MMSP_EINVAL, "src, dst and index must be non-NULL");
  if (!aligned16(src) || !aligned16(dst) || ((uintptr_t)index & 3u))
    return fail(MMSP_EINVAL, "src/dst must be 16-byte aligned and index 4-byte aligned");
  const int64_t bytes = n_rows * row_bytes;
  const char* s0 = static_cast<const char*>(src);
  const char* d0 = static_cast<const char*>(dst);
  if (s0 < d0 + bytes && d0 < s0 + bytes) return fail(MMSP_EINVAL, "src and dst overlap");
  int dev, sms, rc;
  if ((rc = current_device(&dev)) || (rc = device_sms(dev, &sms))) return rc;
  int64_t blocks = (n_rows + 7) / 8;  // 8 warps (rows) per block
  if (blocks > 16LL * sms) blocks = 16LL * sms;
  gather_rows_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), index, n_rows, row_bytes / 16, scatter);
  MMSP_CUDA(cudaGetLastError());
  return ok();
}

int mmsp_shard_rope(const void* src, void* dst, int64_t N, int32_t P, int32_t H, int32_t d, double theta,
                    int32_t interleaved, const int32_t* doc_start, int32_t inverse, void* stream) {
  int rc = check_common(N, P);
  if (rc) return rc;
  if (H < 1) return fail(MMSP_EINVAL, "H must be >= 1");
  if (!(d == 8 || d == 16 || d == 32 || d == 64 || d == 128 || d == 256))
    return fail(MMSP_EINVAL, "d must be one of 8, 16, 32, 64, 128, 256 (got %d)", d);
  if (!(theta > 1.0) || !std::isfinite(theta)) return fail(MMSP_EINVAL, "theta must be finite and > 1");
  if (interleaved != 0 && interleaved != 1) return fail(MMSP_EINVAL, "interleaved must be 0 or 1");
  if (inverse != 0 && inverse != 1) return fail(MMSP_EINVAL, "inverse must be 0 or 1");
  if (!src || !dst) return fail(MMSP_EINVAL, "src and dst must be non-NULL");
  if (!aligned16(src) || !aligned16(dst)) return fail(MMSP_EINVAL, "src and dst must be 16-byte aligned");
  if (doc_start && ((uintptr_t)doc_start & 3u)) return fail(MMSP_EINVAL, "doc_start must be 4-byte aligned");
  const int64_t bytes = N * (int64_t)H * d * 2;
  const char* s0 = static_cast<const char*>(src);
  const char* d0 = static_cast<const char*>(dst);
  if (s0 < d0 + bytes && d0 < s0 + bytes) return fail(MMSP_EINVAL, "src and dst overlap");
  if (N == 0) return ok();
  int dev, sms;
  if ((rc = current_device(&dev)) || (rc = device_sms(dev, &sms))) return rc;
  RopeParams rp;
  for (int i = 0; i < kRopeMaxPairs; ++i) rp.inv_freq[i] = i < d / 2 ? std::pow(theta, -2.0 * i / d) : 0.0;
  rp.N = (int32_t)N;
  rp.P = P;
  rp.H = H;
  rp.inverse = inverse;
  rp.doc_start = doc_start;
  int64_t blocks = (N + 7) / 8;  // 8 warps (rows) per block
  if (blocks > 16LL * sms) blocks = 16LL * sms;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const __nv_bfloat16* sb = static_cast<const __nv_bfloat16*>(src);
  __nv_bfloat16* db = static_cast<__nv_bfloat16*>(dst);
#define MMSP_ROPE(DD)                                                                            \
  case DD:                                                                                       \
    if (interleaved)                                                                             \
      shard_rope_kernel<DD, true><<<(unsigned)blocks, 256, 0, st>>>(rp, sb, db);                 \
    else                                                                                         \
      shard_rope_kernel<DD, false><<<(unsigned)blocks, 256, 0, st>>>(rp, sb, db);                \
    break;
  switch (d) { MMSP_ROPE(8) MMSP_ROPE(16) MMSP_ROPE(32) MMSP_ROPE(64) MMSP_ROPE(128) MMSP_ROPE(256) }
#undef MMSP_ROPE
  MMSP_CUDA(cudaGetLastError());
  return ok();
}

int mmsp_ulysses_transpose(const void* src, void* dst, int64_t S, int32_t H, int32_t P_u, int64_t row_bytes,
                           int32_t unpack, void* stream) {
  if (S < 0) return fail(MMSP_EINVAL, "S must be >= 0 (got %lld)", (long long)S);
  if (H < 1 || P_u < 1 || H % P_u) return fail(MMSP_EINVAL, "need H %% P_u == 0 with H, P_u >= 1 (H=%d P_u=%d)", H, P_u);
  if (row_bytes <= 0 || row_bytes % 16) return fail(MMSP_EINVAL, "row_bytes must be a positive multiple of 16");
  if (unpack != 0 && unpack != 1) return fail(MMSP_EINVAL, "unpack must be 0 or 1");
  if (S == 0) return ok();
  if (!src || !dst) return fail(MMSP_EINVAL, "src and dst must be non-NULL");
  if (!aligned16(src) || !aligned16(dst)) return fail(MMSP_EINVAL, "src and dst must be 16-byte aligned");
  const int64_t run = (int64_t)(H / P_u) * row_bytes;
  if (S > (int64_t(1) << 40) / ((int64_t)H * row_bytes)) return fail(MMSP_EINVAL, "tensor too large");
  const int64_t bytes = S * P_u * run;
  const char* s0 = static_cast<const char*>(src);
  const char* d0 = static_cast<const char*>(dst);
  if (s0 < d0 + bytes && d0 < s0 + bytes) return fail(MMSP_EINVAL, "src and dst overlap");
  int dev, sms, rc;
  if ((rc = current_device(&dev)) || (rc = device_sms(dev, &sms))) return rc;
  int64_t blocks = (S * P_u + 7) / 8;  // 8 warps (runs) per block
  if (blocks > 16LL * sms) blocks = 16LL * sms;
  ulysses_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), S, P_u, run / 16, unpack);
  MMSP_CUDA(cudaGetLastError());
  return ok();
}

int mmsp_lse_merge(const float* o_a, const float* lse_a, const float* o_b, const float* lse_b, float* o_out,
                   float* lse_out, int64_t rows, int32_t H, int32_t d, void* stream) {
  if (rows < 0 || H < 1) return fail(MMSP_EINVAL, "rows must be >= 0 and H >= 1");
  if (!(d == 4 || d == 8 || d == 16 || d == 32 || d == 64 || d == 128))
    return fail(MMSP_EINVAL, "d must be one of 4, 8, 16, 32, 64, 128 (got %d)", d);
  if (!o_a || !lse_a || !o_b || !lse_b || !o_out || !lse_out) return fail(MMSP_EINVAL, "NULL pointer");
  if (!aligned16(o_a) || !aligned16(o_b) || !aligned16(o_out))
    return fail(MMSP_EINVAL, "o_a, o_b, o_out must be 16-byte aligned");
  if (((uintptr_t)lse_a | (uintptr_t)lse_b | (uintptr_t)lse_out) & 3u) return fail(MMSP_EINVAL, "lse pointers must be 4-byte aligned");
  const int64_t total = rows * H;
  if (total == 0) return ok();
  int dev, sms, rc;
  if ((rc = current_device(&dev)) || (rc = device_sms(dev, &sms))) return rc;
  int64_t warps = (total + 31) / 32;
  int64_t blocks = (warps + 7) / 8;
  if (blocks > 8LL * sms) blocks = 8LL * sms;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
#define MMSP_MERGE(DD) \
  case DD:             \
    lse_merge_kernel<DD><<<(unsigned)blocks, 256, 0, st>>>(o_a, lse_a, o_b, lse_b, o_out, lse_out, total); break;
  switch (d) { MMSP_MERGE(4) MMSP_MERGE(8) MMSP_MERGE(16) MMSP_MERGE(32) MMSP_MERGE(64) MMSP_MERGE(128) }
#undef MMSP_MERGE
  MMSP_CUDA(cudaGetLastError());
  return ok();
}

}  // extern "C"

namespace {
// One forward variant: shared-memory opt-in once per device, then launch.
template <int D, bool DOC>
int launch_fwd(int dev, int vi, int64_t grid, cudaStream_t st, const CUtensorMap& tq, const CUtensorMap& tk,
               const CUtensorMap& tv, const fwd::Params& p) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_dev[dev].fwd_attr[vi]) {
      // The kernel's warpgroups re-split the launch's registers; a build
      // that launches with fewer per thread would make the split wait.
      cudaFuncAttributes fa;
      MMSP_CUDA(cudaFuncGetAttributes(&fa, fwd::attn_fwd_kernel<D, DOC>));
      if (fa.numRegs < fwd::kRegLaunch)
        return fail(MMSP_ECUDA, "forward kernel built with %d registers per thread, the register split needs %d",
                    fa.numRegs, fwd::kRegLaunch);
      MMSP_CUDA(cudaFuncSetAttribute(fwd::attn_fwd_kernel<D, DOC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     fwd::Smem<D>::ALLOC));
      g_dev[dev].fwd_attr[vi] = true;
    }
  }
  fwd::attn_fwd_kernel<D, DOC><<<(unsigned)grid, fwd::kThreads, fwd::Smem<D>::ALLOC, st>>>(tq, tk, tv, p);
  MMSP_CUDA(cudaGetLastError());
  return MMSP_OK;
}
}  // namespace

extern "C" {

int mmsp_attn_fwd(const void* q, const void* k, const void* v, int64_t N, int32_t P, int32_t Hq, int32_t Hkv,
                  int32_t d, float scale, int32_t causal, int32_t step_begin, int32_t step_end, int32_t rank_begin,
                  int32_t rank_end, float* o_acc, float* lse, void* o_out, uint32_t flags, const int32_t* doc_start,
                  void* stream) {
  int rc = check_common(N, P);
  if (rc) return rc;
  if ((rc = check_ranks(P, rank_begin, rank_end))) return rc;
  if ((rc = check_heads(Hq, Hkv, d))) return rc;
  if (doc_start && causal != 1) return fail(MMSP_EINVAL, "doc_start needs causal = 1");
  if (doc_start && ((uintptr_t)doc_start & 3u)) return fail(MMSP_EINVAL, "doc_start must be 4-byte aligned");
  if (flags & ~(MMSP_ACCUMULATE | MMSP_FINALIZE)) return fail(MMSP_EINVAL, "unknown flags 0x%x", flags);
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(MMSP_EINVAL, "scale must be finite and > 0");
  if (causal != 0 && causal != 1) return fail(MMSP_EINVAL, "causal must be 0 or 1");
  if (step_begin < 0 || step_end < step_begin || step_end > P)
    return fail(MMSP_EINVAL, "need 0 <= step_begin <= step_end <= P (got %d, %d, P=%d)", step_begin, step_end, P);
  if (!q || !k || !v || !lse) return fail(MMSP_EINVAL, "q, k, v and lse must be non-NULL");
  if ((flags & MMSP_ACCUMULATE) && !o_acc) return fail(MMSP_EINVAL, "MMSP_ACCUMULATE needs o_acc");
  if ((flags & MMSP_FINALIZE) && !o_out) return fail(MMSP_EINVAL, "MMSP_FINALIZE needs o_out");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(lse) || (o_acc && !aligned16(o_acc)) ||
      (o_out && !aligned16(o_out)))
    return fail(MMSP_EINVAL, "all tensors must be 16-byte aligned");
  if (N == 0) return ok();
  int dev, sms;
  if ((rc = current_device(&dev)) || (rc = device_sms(dev, &sms)) || (rc = get_encode())) return rc;
  CUtensorMap tq, tk, tv;
  if ((rc = tmap_rows_heads(&tq, q, N, Hq, d)) || (rc = tmap_rows_heads(&tk, k, N, Hkv, d)) ||
      (rc = tmap_rows_heads(&tv, v, N, Hkv, d)))
    return rc;
  fwd::Params p;
  p.P = P;
  p.rank_begin = rank_begin;
  p.n_ranks = rank_end - rank_begin;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.C = N / (2 * (int64_t)P);
  p.nblk = (int32_t)((p.C + 255) / 256);
  p.causal = causal;
  p.step_begin = step_begin;
  p.step_end = step_end;
  p.accumulate = (flags & MMSP_ACCUMULATE) ? 1 : 0;
  p.finalize = (flags & MMSP_FINALIZE) ? 1 : 0;
  p.n_items = 2LL * p.n_ranks * p.nblk * Hq;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o_acc = o_acc;
  p.lse = lse;
  p.o_out = static_cast<__nv_bfloat16*>(o_out);
  p.doc_start = doc_start;
  p.wait_cap = kWaitCapCycles;
  const int64_t grid = p.n_items < sms ? p.n_items : sms;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int vi = (d == 128 ? 2 : 0) + (doc_start ? 1 : 0);
  if (d == 128)
    rc = doc_start ? launch_fwd<128, true>(dev, vi, grid, st, tq, tk, tv, p)
                   : launch_fwd<128, false>(dev, vi, grid, st, tq, tk, tv, p);
  else
    rc = doc_start ? launch_fwd<64, true>(dev, vi, grid, st, tq, tk, tv, p)
                   : launch_fwd<64, false>(dev, vi, grid, st, tq, tk, tv, p);
  if (rc) return rc;
  return ok();
}

int mmsp_device_status(void* stream) {
  MMSP_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  MMSP_CUDA(cudaGetLastError());
  int flag = 0;
  MMSP_CUDA(cudaMemcpyFromSymbol(&flag, g_timeout_flag, sizeof(int)));
  if (flag) {
    const int zero = 0;
    MMSP_CUDA(cudaMemcpyToSymbol(g_timeout_flag, &zero, sizeof(int)));
    if (flag == 2) return fail(MMSP_ECUDA, "a kernel found its shared memory base misaligned and did nothing");
    if (flag == 3) return fail(MMSP_EINVAL, "an index array held a value out of range (those rows were skipped)");
    return fail(MMSP_ETIMEOUT, "a bounded device-side wait gave up");
  }
  return ok();
}

}  // extern "C"

namespace {
__global__ void selftest_wait_kernel(long long max_cycles) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_word;
  if (threadIdx.x == 0) {
    mmsp::mbar_init(mmsp::smem_u32(&bar), 1);
    abort_word = 0;
    mmsp::fence_barrier_init();
  }
  __syncthreads();
  // Nobody arrives: the wait must give up and record the timeout.
  mmsp::mbar_wait(mmsp::smem_u32(&bar), 0, &abort_word, max_cycles);
}
}  // namespace

extern "C" int mmsp_selftest_bounded_wait(int64_t max_cycles, void* stream) {
  if (max_cycles < 1 || max_cycles > (int64_t(1) << 31))
    return fail(MMSP_EINVAL, "max_cycles must be in [1, 2^31]");
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>((long long)max_cycles);
  MMSP_CUDA(cudaGetLastError());
  return ok();
}

namespace {
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct BwdLayout {
  int64_t C, Cp;
  size_t vec_bytes, total;
};

// Backward scratch: LSE*log2(e) and D per head in padded rows (two arrays).
BwdLayout bwd_layout(int64_t N, int32_t P, int32_t Hq, int32_t d) {
  (void)d;
  BwdLayout L;
  L.C = N / (2 * (int64_t)P);
  L.Cp = (L.C + 127) / 128 * 128;
  L.vec_bytes = align256((size_t)Hq * 2 * P * L.Cp * sizeof(float));
  L.total = 2 * L.vec_bytes;
  return L;
}
}  // namespace

extern "C" size_t mmsp_bwd_workspace_bytes(int64_t N, int32_t P, int32_t Hq, int32_t d) {
  if (N <= 0 || P < 1 || Hq < 1 || d < 1 || N % (2 * (int64_t)P)) return 0;
  return bwd_layout(N, P, Hq, d).total;
}

namespace {
// Shared checks of the backward stages (sizes, scale, workspace).
int bwd_check(int64_t N, int32_t P, int32_t Hq, int32_t Hkv, int32_t d, float scale, int32_t causal,
              int32_t rank_begin, int32_t rank_end, const void* workspace, size_t workspace_bytes,
              const int32_t* doc_start = nullptr) {
  int rc = check_common(N, P);
  if (rc) return rc;
  if ((rc = check_ranks(P, rank_begin, rank_end))) return rc;
  if ((rc = check_heads(Hq, Hkv, d))) return rc;
  if (d != 128) return fail(MMSP_EUNSUPPORTED, "the backward supports d = 128 (got %d)", d);
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(MMSP_EINVAL, "scale must be finite and > 0");
  if (causal != 0 && causal != 1) return fail(MMSP_EINVAL, "causal must be 0 or 1");
  if (doc_start && causal != 1) return fail(MMSP_EINVAL, "doc_start needs causal = 1");
  if (doc_start && ((uintptr_t)doc_start & 3u)) return fail(MMSP_EINVAL, "doc_start must be 4-byte aligned");
  if (N == 0) return MMSP_OK;
  const BwdLayout Lw = bwd_layout(N, P, Hq, d);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(MMSP_EINVAL, "workspace must be non-NULL and 256-byte aligned");
  if (workspace_bytes < Lw.total)
    return fail(MMSP_EINVAL, "workspace too small: %zu < %zu bytes", workspace_bytes, Lw.total);
  return MMSP_OK;
}

bool all_aligned16(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (p && !aligned16(p)) return false;
  return true;
}

// Parameters and tensor maps of the two tcgen05 backward kernels.
int bwd_setup(const void* q, const void* k, const void* v, const void* dout, int64_t N, int32_t P, int32_t Hq,
              int32_t Hkv, int32_t d, float scale, int32_t causal, int32_t rank_begin, int32_t rank_end,
              const void* workspace, bwd::Params* p,
              CUtensorMap* tq, CUtensorMap* tk, CUtensorMap* tv, CUtensorMap* tdo, int* sms) {
  int dev, rc;
  if ((rc = current_device(&dev)) || (rc = device_sms(dev, sms)) || (rc = get_encode())) return rc;
  if ((rc = tmap_rows_heads(tq, q, N, Hq, d)) || (rc = tmap_rows_heads(tk, k, N, Hkv, d)) ||
      (rc = tmap_rows_heads(tv, v, N, Hkv, d)) || (rc = tmap_rows_heads(tdo, dout, N, Hq, d)))
    return rc;
  const BwdLayout Lw = bwd_layout(N, P, Hq, d);
  const char* ws = static_cast<const char*>(workspace);
  *p = bwd::Params{};
  p->P = P;
  p->rank_begin = rank_begin;
  p->n_ranks = rank_end - rank_begin;
  p->Hq = Hq;
  p->Hkv = Hkv;
  p->G = Hq / Hkv;
  p->C = Lw.C;
  p->Cp = Lw.Cp;
  p->ntiles = (int32_t)(Lw.Cp / 128);
  p->causal = causal;
  p->n_units = 2LL * p->n_ranks * p->ntiles * Hkv;
  p->n_items = 2LL * p->n_ranks * p->ntiles * Hq;
  p->scale_log2 = scale * 1.4426950408889634f;
  p->scale = scale;
  p->lse2t = reinterpret_cast<const float*>(ws);
  p->dt = reinterpret_cast<const float*>(ws + Lw.vec_bytes);
  p->wait_cap = kWaitCapCycles;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_dev[dev].bwd_attr[1]) {
    MMSP_CUDA(cudaFuncSetAttribute(bwd::attn_bwd_dkdv_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   bwd::SmemKV::ALLOC));
    MMSP_CUDA(cudaFuncSetAttribute(bwd::attn_bwd_dkdv_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   bwd::SmemKV::ALLOC));
    MMSP_CUDA(cudaFuncSetAttribute(bwd::attn_bwd_dq_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   bwd::SmemQ::ALLOC));
    MMSP_CUDA(cudaFuncSetAttribute(bwd::attn_bwd_dq_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   bwd::SmemQ::ALLOC));
    g_dev[dev].bwd_attr[1] = true;
  }
  return MMSP_OK;
}
}  // namespace

extern "C" int mmsp_attn_bwd_prepare(const void* o, const void* dout, const float* lse, int64_t N, int32_t P,
                                     int32_t Hq, int32_t d, int32_t rank_begin, int32_t rank_end, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  int rc = bwd_check(N, P, Hq, 1, d, 1.f, 1, rank_begin, rank_end, workspace, workspace_bytes);
  if (rc) return rc;
  if (!o || !dout || !lse) return fail(MMSP_EINVAL, "o, dout and lse must be non-NULL");
  if (!all_aligned16({o, dout, lse})) return fail(MMSP_EINVAL, "all tensors must be 16-byte aligned");
  if (N == 0) return ok();
  int dev, sms;
  if ((rc = current_device(&dev)) || (rc = device_sms(dev, &sms))) return rc;
  const BwdLayout Lw = bwd_layout(N, P, Hq, d);
  char* ws = static_cast<char*>(workspace);
  const int64_t pre_warps = (int64_t)(rank_end - rank_begin) * 2 * Lw.Cp * Hq;
  int64_t pre_blocks = (pre_warps + 7) / 8;
  if (pre_blocks > 16LL * sms) pre_blocks = 16LL * sms;
  bwd::bwd_pre_kernel<<<(unsigned)pre_blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse,
      reinterpret_cast<float*>(ws), reinterpret_cast<float*>(ws + Lw.vec_bytes), rank_begin, rank_end - rank_begin, Hq,
      Lw.C, Lw.Cp);
  MMSP_CUDA(cudaGetLastError());
  return ok();
}

extern "C" int mmsp_attn_bwd_dkdv(const void* q, const void* k, const void* v, const void* dout, int64_t N,
                                  int32_t P, int32_t Hq, int32_t Hkv, int32_t d, float scale, int32_t causal,
                                  int32_t rank_begin, int32_t rank_end, void* dk, void* dv, const void* workspace,
                                  size_t workspace_bytes, const int32_t* doc_start, void* stream) {
  int rc = bwd_check(N, P, Hq, Hkv, d, scale, causal, rank_begin, rank_end, workspace, workspace_bytes, doc_start);
  if (rc) return rc;
  if (!q || !k || !v || !dout || !dk || !dv) return fail(MMSP_EINVAL, "q, k, v, dout, dk, dv must be non-NULL");
  if (!all_aligned16({q, k, v, dout, dk, dv})) return fail(MMSP_EINVAL, "all tensors must be 16-byte aligned");
  if (N == 0) return ok();
  bwd::Params p;
  CUtensorMap tq, tk, tv, tdo;
  int sms;
  if ((rc = bwd_setup(q, k, v, dout, N, P, Hq, Hkv, d, scale, causal, rank_begin, rank_end, workspace, &p, &tq, &tk,
                      &tv, &tdo, &sms)))
    return rc;
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.doc_start = doc_start;
  const int64_t grid = p.n_units < sms ? p.n_units : sms;
  if (doc_start)
    bwd::attn_bwd_dkdv_kernel<true><<<(unsigned)grid, bwd::kThreads, bwd::SmemKV::ALLOC,
                                      static_cast<cudaStream_t>(stream)>>>(tq, tk, tv, tdo, p);
  else
    bwd::attn_bwd_dkdv_kernel<false><<<(unsigned)grid, bwd::kThreads, bwd::SmemKV::ALLOC,
                                       static_cast<cudaStream_t>(stream)>>>(tq, tk, tv, tdo, p);
  MMSP_CUDA(cudaGetLastError());
  return ok();
}

extern "C" int mmsp_attn_bwd_dq(const void* q, const void* k, const void* v, const void* dout, int64_t N, int32_t P,
                                int32_t Hq, int32_t Hkv, int32_t d, float scale, int32_t causal, int32_t rank_begin,
                                int32_t rank_end, void* dq, float* dq_acc_opt, const void* workspace,
                                size_t workspace_bytes, const int32_t* doc_start, void* stream) {
  int rc = bwd_check(N, P, Hq, Hkv, d, scale, causal, rank_begin, rank_end, workspace, workspace_bytes, doc_start);
  if (rc) return rc;
  if (!q || !k || !v || !dout || !dq) return fail(MMSP_EINVAL, "q, k, v, dout, dq must be non-NULL");
  if (!all_aligned16({q, k, v, dout, dq, dq_acc_opt})) return fail(MMSP_EINVAL, "all tensors must be 16-byte aligned");
  if (N == 0) return ok();
  bwd::Params p;
  CUtensorMap tq, tk, tv, tdo;
  int sms;
  if ((rc = bwd_setup(q, k, v, dout, N, P, Hq, Hkv, d, scale, causal, rank_begin, rank_end, workspace, &p, &tq, &tk,
                      &tv, &tdo, &sms)))
    return rc;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dq_acc = dq_acc_opt;
  p.doc_start = doc_start;
  const int64_t grid = p.n_items < sms ? p.n_items : sms;
  if (doc_start)
    bwd::attn_bwd_dq_kernel<true><<<(unsigned)grid, bwd::kThreads, bwd::SmemQ::ALLOC,
                                    static_cast<cudaStream_t>(stream)>>>(tq, tk, tv, tdo, p);
  else
    bwd::attn_bwd_dq_kernel<false><<<(unsigned)grid, bwd::kThreads, bwd::SmemQ::ALLOC,
                                     static_cast<cudaStream_t>(stream)>>>(tq, tk, tv, tdo, p);
  MMSP_CUDA(cudaGetLastError());
  return ok();
}

extern "C" int mmsp_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                             const float* lse, int64_t N, int32_t P, int32_t Hq, int32_t Hkv, int32_t d, float scale,
                             int32_t causal, void* dq, void* dk, void* dv, float* dq_acc_opt, void* workspace,
                             size_t workspace_bytes, const int32_t* doc_start, void* stream) {
  int rc = bwd_check(N, P, Hq, Hkv, d, scale, causal, 0, P, workspace, workspace_bytes, doc_start);
  if (rc) return rc;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv)
    return fail(MMSP_EINVAL, "q, k, v, o, dout, lse, dq, dk, dv must be non-NULL");
  if (!all_aligned16({q, k, v, o, dout, lse, dq, dk, dv, dq_acc_opt}))
    return fail(MMSP_EINVAL, "all tensors must be 16-byte aligned");
  if (N == 0) return ok();
  if ((rc = mmsp_attn_bwd_prepare(o, dout, lse, N, P, Hq, d, 0, P, workspace, workspace_bytes, stream))) return rc;
  if ((rc = mmsp_attn_bwd_dkdv(q, k, v, dout, N, P, Hq, Hkv, d, scale, causal, 0, P, dk, dv, workspace,
                               workspace_bytes, doc_start, stream)))
    return rc;
  return mmsp_attn_bwd_dq(q, k, v, dout, N, P, Hq, Hkv, d, scale, causal, 0, P, dq, dq_acc_opt, workspace,
                          workspace_bytes, doc_start, stream);
}

// ---------------------------------------------------------------------------
// Allocation-free backward: the scratch of mmsp_attn_bwd in a file-scope
// device array, shared by every call on a device.
namespace {
__device__ __align__(256) unsigned char g_bwd_scratch[MMSP_NOALLOC_SCRATCH_BYTES];

void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_bwd_scratch on the current device (host code only
// sees a host-side stand-in for the symbol; passing that to a kernel would
// be wrong). Looked up again on every call made outside stream capture, so
// that a context torn down and re-created (cudaDeviceReset) cannot leave a
// stale address behind; a call under capture reuses the address of the
// last uncaptured call on the device (the lookup allocates nothing either
// way).
int scratch_address(int dev, cudaStream_t st, void** out) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(st, &cs);
  if (e != cudaSuccess) return fail(MMSP_ECUDA, "cudaStreamIsCapturing failed: %s", cudaGetErrorString(e));
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (cs == cudaStreamCaptureStatusNone || !g_scratch_ptr[dev]) {
    if (cs != cudaStreamCaptureStatusNone)
      return fail(MMSP_EINVAL, "the first mmsp_attn_bwd_noalloc call on a device must not be under stream capture");
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_bwd_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(MMSP_ECUDA, "cudaGetSymbolAddress(scratch) failed: %s", cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MMSP_OK;
}
}  // namespace

extern "C" int mmsp_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                     const float* lse, int64_t N, int32_t P, int32_t Hq, int32_t Hkv, int32_t d,
                                     float scale, int32_t causal, void* dq, void* dk, void* dv, float* dq_acc_opt,
                                     const int32_t* doc_start, void* stream) {
  int rc = check_common(N, P);
  if (rc) return rc;
  if ((rc = check_heads(Hq, Hkv, d))) return rc;
  if (N == 0) return mmsp_attn_bwd(q, k, v, o, dout, lse, N, P, Hq, Hkv, d, scale, causal, dq, dk, dv, dq_acc_opt,
                                   nullptr, 0, doc_start, stream);
  const size_t need = mmsp_bwd_workspace_bytes(N, P, Hq, d);
  if (need > (size_t)MMSP_NOALLOC_SCRATCH_BYTES)
    return fail(MMSP_EINVAL, "sizes need %zu bytes of scratch; mmsp_attn_bwd_noalloc holds at most %zu (use "
                "mmsp_attn_bwd with a caller workspace)", need, (size_t)MMSP_NOALLOC_SCRATCH_BYTES);
  int dev;
  if ((rc = current_device(&dev))) return rc;
  void* scratch = nullptr;
  if ((rc = scratch_address(dev, static_cast<cudaStream_t>(stream), &scratch))) return rc;
  return mmsp_attn_bwd(q, k, v, o, dout, lse, N, P, Hq, Hkv, d, scale, causal, dq, dk, dv, dq_acc_opt, scratch,
                       (size_t)MMSP_NOALLOC_SCRATCH_BYTES, doc_start, stream);
}
