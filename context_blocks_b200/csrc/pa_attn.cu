// C ABI of the blockwise attention library: argument checks, TMA tensor-map
// encoding and kernel launches.  See include/pa_attn.h for the contract.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <algorithm>
#include <atomic>
#include <mutex>

#include "attn_fwd.cuh"
#include "quantize.cuh"
#include "fwd_common.cuh"
#include "lse_merge.cuh"
#include "residual_diff.cuh"
#include "pa_attn.h"

namespace pa {

// Device status word: kernels record the first device-side error here.
__device__ int g_status = 0;

// Scratch for pa_attn_chunks_noalloc: the per-chunk partial outputs and LSEs
// live here instead of in memory the caller or the library allocates.  Every
// GPU that loads the library holds these 32 MiB until the process exits.
constexpr unsigned long long kNoAllocScratchBytes = 32ull << 20;
constexpr int kNoAllocMaxChunks = 64;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

__global__ void timeout_probe_kernel(unsigned long long limit_ns, int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_word;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_word = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`; the bounded wait gives up after limit_ns.
  mbar_wait(smem_u32(&bar), 0, &abort_word, status, kStatusTimeout, limit_ns);
}

}  // namespace pa

namespace {

constexpr int kDefaultWaitLimitMs = 5000;
constexpr int kMaxDevices = 64;

// Limit of every device-side barrier wait, in nanoseconds (pa_set_wait_limit_ms).
std::atomic<unsigned long long> g_wait_limit_ns{static_cast<unsigned long long>(kDefaultWaitLimitMs) * 1000000ull};

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(PA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

struct DeviceState {
  bool ready = false;
  bool supported = false;
  int sm_count = 0;
  int* status = nullptr;  // device address of pa::g_status
  unsigned char* noalloc_scratch = nullptr;  // device address of pa::g_noalloc_scratch
  bool fwd_attr[5] = {};  // d = 64, d = 128, e4m3 d = 128, accumulate d = 64, accumulate d = 128
};


std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

// Per-device set-up, once: capability check, SM count, status-word address.
int device_state(int dev, DeviceState** out) {
  if (dev < 0 || dev >= kMaxDevices) return fail(PA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& s = g_dev[dev];
  if (!s.ready) {
    int major = 0, minor = 0, sms = 0;
    cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    s.supported = (major == 10 && minor == 0);
    s.sm_count = sms;
    if (s.supported) {
      void* addr = nullptr;
      e = cudaGetSymbolAddress(&addr, pa::g_status);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status)");
      s.status = static_cast<int*>(addr);
      // In host code the array's name is only a host-side stand-in: the
      // kernels must be given this device address instead.
      void* scratch = nullptr;
      e = cudaGetSymbolAddress(&scratch, pa::g_noalloc_scratch);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(noalloc scratch)");
      s.noalloc_scratch = static_cast<unsigned char*>(scratch);
    }
    s.ready = true;
  }
  if (!s.supported) return fail(PA_ERR_UNSUPPORTED, "device %d is not sm_100 (B200)", dev);
  *out = &s;
  return PA_OK;
}

// The pointer must be device (or managed) memory of the current device.
int check_device_ptr(const void* ptr, const char* name, int* dev_out) {
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, ptr);
  if (e != cudaSuccess) return cuda_fail(e, "cudaPointerGetAttributes");
  if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
    return fail(PA_ERR_INVALID_ARG, "%s is not device memory", name);
  int cur = 0;
  e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (attr.device != cur)
    return fail(PA_ERR_INVALID_ARG, "%s lives on device %d, current device is %d", name, attr.device, cur);
  *dev_out = cur;
  return PA_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlap(const void* a, uint64_t na, const void* b, uint64_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D map over a [BH, N, d] bf16 tensor: box of 64 head-dim elements x
// box_rows rows x 1, 128-byte swizzle, zero fill outside the tensor.
// 3-D map (d, N, B*H) with 128-byte swizzled boxes of one 128-byte row of d by
// box_rows rows: 64 bf16 or (fp8) 128 one-byte elements per row.
int encode_map(CUtensorMap* map, const void* ptr, int d, int n_rows, int bh, int box_rows, bool fp8 = false) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled entry point not available");
  const int eb = fp8 ? 1 : 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n_rows),
                        static_cast<cuuint64_t>(bh)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * eb,
                           static_cast<cuuint64_t>(n_rows) * static_cast<cuuint64_t>(d) * eb};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / eb), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(ptr), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", int(r));
  return PA_OK;
}

// Running state of an accumulating launch (pa_attn_fwd_accum); acc_o null
// for an ordinary launch.
struct AccArgs {
  float* acc_o = nullptr;
  float* acc_lse = nullptr;
  int flags = 0;
};

// Single-CTA forward over n_chunks K/V chunks (n_chunks = 1 for one chunk).
// kFp8: e4m3 Q/K/V with dequantisation scales; qk_scale multiplies the logits
// (on top of `scale`) and o_scale the output.
template <int D, bool kFp8 = false>
int launch_fwd(DeviceState* st, const void* q, const void* const* k, const void* const* v, const int* nk,
               int n_chunks, void* o, float* lse, int BH, int Nq, float scale, cudaStream_t stream,
               float qk_scale = 1.f, float o_scale = 1.f, const float* const* dscales = nullptr,
               const AccArgs& acc = AccArgs()) {
  using L = pa::single::FwdLayout<D, kFp8>;
  CUtensorMap tq;
  pa::single::KvChunks kv;
  int rc;
  if ((rc = encode_map(&tq, q, D, Nq, BH, pa::kBM, kFp8)) != PA_OK) return rc;
  long long nk_total = 0, tiles_total = 0;
  for (int c = 0; c < n_chunks; ++c) {
    if ((rc = encode_map(&kv.k[c], k[c], D, nk[c], BH, pa::kBN, kFp8)) != PA_OK) return rc;
    if ((rc = encode_map(&kv.v[c], v[c], D, nk[c], BH, pa::kBN, kFp8)) != PA_OK) return rc;
    kv.nk[c] = nk[c];
    kv.tiles[c] = (nk[c] + pa::kBN - 1) / pa::kBN;
    kv.tile_start[c] = static_cast<int>(tiles_total);
    nk_total += nk[c];
    tiles_total += kv.tiles[c];
  }
  for (int c = n_chunks; c < pa::single::kMaxChunks; ++c) {
    kv.nk[c] = 0;
    kv.tiles[c] = 0;
    kv.tile_start[c] = 0x7fffffff;  // never reached by a tile index
  }
  kv.n_chunks = n_chunks;
  if (nk_total > 0x7fffffffLL) return fail(PA_ERR_UNSUPPORTED, "more than 2^31 keys in one call");
  // Accumulate mode is its own instantiation (bf16 only), so that the plain
  // forward carries none of its code.
  const bool accum = acc.acc_o != nullptr;
  if (kFp8 && accum) return fail(PA_ERR_UNSUPPORTED, "accumulate mode takes bf16 inputs");
  auto kern = pa::single::attn_fwd_kernel<D, kFp8, false>;
  if constexpr (!kFp8)
    if (accum) kern = pa::single::attn_fwd_kernel<D, false, true>;
  const int slot = kFp8 ? 2 : (D == 64 ? 0 : 1) + (accum ? 3 : 0);
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!st->fwd_attr[slot]) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAllocBytes);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
      // The kernel's register split assumes this launch allocation; with any
      // other count its setmaxnreg.inc could wait for ever.
      cudaFuncAttributes fa;
      e = cudaFuncGetAttributes(&fa, kern);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes");
      if (fa.numRegs != pa::single::kLaunchRegs)
        return fail(PA_ERR_UNSUPPORTED, "forward kernel built with %d registers per thread, the register split "
                    "needs %d", fa.numRegs, pa::single::kLaunchRegs);
      st->fwd_attr[slot] = true;
    }
  }
  pa::FwdParams prm;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.Nq = Nq;
  prm.Nk = static_cast<int>(nk_total);
  prm.n_kv_tiles = static_cast<int>(tiles_total);
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.status = st->status;
  prm.timeout_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  prm.qk_scale = qk_scale;
  prm.o_scale = o_scale;
  prm.dscale_q = dscales ? dscales[0] : nullptr;
  prm.dscale_k = dscales ? dscales[1] : nullptr;
  prm.dscale_v = dscales ? dscales[2] : nullptr;
  prm.acc_o = acc.acc_o;
  prm.acc_lse = acc.acc_lse;
  prm.acc_flags = acc.flags;
  // Persistent grid: one CTA per SM (shared memory and tensor memory allow
  // no more), each walking the (b*h, 256-row block) items.
  prm.blocks_per_bh = (Nq + pa::kQTiles * pa::kBM - 1) / (pa::kQTiles * pa::kBM);
  const long long items = static_cast<long long>(prm.blocks_per_bh) * BH;
  if (items > 0x7fffffffLL) return fail(PA_ERR_UNSUPPORTED, "too many query blocks");
  prm.items = static_cast<int>(items);
  const unsigned grid = static_cast<unsigned>(std::min<long long>(items, st->sm_count));
  kern<<<grid, pa::single::kFwdThreads, L::kAllocBytes, stream>>>(tq, kv, prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attn_fwd launch");
  return PA_OK;
}

// The bf16 forward for head dim d (64 or 128).
int launch_bf16(DeviceState* st, int d, const void* q, const void* const* k, const void* const* v, const int* nk,
                int n_chunks, void* o, float* lse, int BH, int Nq, float scale, cudaStream_t stream,
                const AccArgs& acc = AccArgs()) {
  if (d == 64) return launch_fwd<64>(st, q, k, v, nk, n_chunks, o, lse, BH, Nq, scale, stream, 1.f, 1.f, nullptr, acc);
  return launch_fwd<128>(st, q, k, v, nk, n_chunks, o, lse, BH, Nq, scale, stream, 1.f, 1.f, nullptr, acc);
}

template <int D>
int launch_merge(DeviceState* st, const void* o_parts, const float* lse_parts, int n_parts, void* o,
                 float* lse, long long rows, cudaStream_t stream) {
  constexpr int kRpb = pa::kMergeThreads / (D / 8);
  long long blocks = (rows + kRpb - 1) / kRpb;
  const long long cap = static_cast<long long>(st->sm_count) * 8;
  if (blocks > cap) blocks = cap;
  pa::lse_merge_kernel<D><<<static_cast<unsigned>(blocks), pa::kMergeThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(o_parts), lse_parts, n_parts, static_cast<__nv_bfloat16*>(o), lse,
      rows);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "lse_merge launch");
  return PA_OK;
}

}  // namespace

namespace {

// Host-side checks of one forward call (no CUDA API touched): pointers, sizes,
// alignment, and that no output overlaps an input or another output.
// o_elem_bytes is 2 for a bf16 output, 4 for the fp32 running state of an
// accumulating call; o2 is a second output of o's shape (the bf16 output of a
// final fold), or null.
int host_fwd_checks(const void* q, const void* k, const void* v, const void* o, const float* lse, int B, int H,
                    int Nq, int Nk, int d, float scale, int in_elem_bytes = 2, int o_elem_bytes = 2,
                    const void* o2 = nullptr) {
  if (!q || !k || !v || !o || !lse) return fail(PA_ERR_INVALID_ARG, "null pointer argument");
  if (B < 1 || H < 1) return fail(PA_ERR_INVALID_ARG, "B and H must be >= 1 (got %d, %d)", B, H);
  if (Nq < 0) return fail(PA_ERR_INVALID_ARG, "Nq must be >= 0 (got %d)", Nq);
  if (Nk < 1) return fail(PA_ERR_INVALID_ARG, "Nk must be >= 1 (got %d)", Nk);
  if (!std::isfinite(scale) || !(scale > 0.f)) return fail(PA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (d != 64 && d != 128) return fail(PA_ERR_UNSUPPORTED, "d must be 64 or 128 (got %d)", d);
  const long long bh = static_cast<long long>(B) * H;
  if (bh > 65535) return fail(PA_ERR_UNSUPPORTED, "B*H must be <= 65535 (got %lld)", bh);
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || (o2 && !aligned(o2, 16)))
    return fail(PA_ERR_MISALIGNED, "q, k, v and o must be 16-byte aligned");
  if (!aligned(lse, 4)) return fail(PA_ERR_MISALIGNED, "lse must be 4-byte aligned");
  if (Nq == 0) return PA_OK;
  const uint64_t qbytes = static_cast<uint64_t>(bh) * Nq * d * in_elem_bytes;
  const uint64_t kbytes = static_cast<uint64_t>(bh) * Nk * d * in_elem_bytes;
  const uint64_t obytes = static_cast<uint64_t>(bh) * Nq * d * o_elem_bytes;
  const uint64_t o2bytes = static_cast<uint64_t>(bh) * Nq * d * 2;
  const uint64_t lbytes = static_cast<uint64_t>(bh) * Nq * 4;
  const void* ins[3] = {q, k, v};
  const uint64_t in_bytes[3] = {qbytes, kbytes, kbytes};
  for (int i = 0; i < 3; ++i)
    if (overlap(ins[i], in_bytes[i], o, obytes) || overlap(ins[i], in_bytes[i], lse, lbytes) ||
        (o2 && overlap(ins[i], in_bytes[i], o2, o2bytes)))
      return fail(PA_ERR_INVALID_ARG, "outputs overlap an input");
  if (overlap(o, obytes, lse, lbytes)) return fail(PA_ERR_INVALID_ARG, "o and lse overlap");
  if (o2 && (overlap(o2, o2bytes, o, obytes) || overlap(o2, o2bytes, lse, lbytes)))
    return fail(PA_ERR_INVALID_ARG, "o overlaps the running state");
  return PA_OK;
}

// Every pointer must be device memory of the current device; on PA_OK *st is
// that device's state.  Each distinct pointer is queried once.
int device_checks(const void* const* ptrs, const char* const* names, int n, DeviceState** st) {
  (void)cudaGetLastError();
  int dev = 0, rc;
  for (int i = 0; i < n; ++i) {
    bool seen = false;
    for (int j = 0; j < i && !seen; ++j) seen = (ptrs[j] == ptrs[i]);
    if (!seen && (rc = check_device_ptr(ptrs[i], names[i], &dev)) != PA_OK) return rc;
  }
  return device_state(dev, st);
}

// Host and device checks of a one-chunk forward.  On PA_OK, *st is the current
// device's state, or null when there is nothing to do (Nq == 0).
int check_fwd_args(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq, int Nk,
                   int d, float scale, DeviceState** st, int in_elem_bytes = 2) {
  *st = nullptr;
  int rc = host_fwd_checks(q, k, v, o, lse, B, H, Nq, Nk, d, scale, in_elem_bytes);
  if (rc != PA_OK || Nq == 0) return rc;
  const void* ptrs[5] = {q, k, v, o, lse};
  const char* names[5] = {"q", "k", "v", "o", "lse"};
  return device_checks(ptrs, names, 5, st);
}

// The same for a table of chunks: every chunk's host checks first, so no CUDA
// call is made for a bad table, then each distinct pointer once.
int check_chunk_args(const void* q, const void* const* k_chunks, const void* const* v_chunks, const int* nk_chunks,
                     int n_chunks, int max_chunks, void* o, float* lse, int B, int H, int Nq, int d, float scale,
                     DeviceState** st) {
  *st = nullptr;
  if (!q || !k_chunks || !v_chunks || !nk_chunks || !o || !lse)
    return fail(PA_ERR_INVALID_ARG, "null pointer argument");
  if (n_chunks < 1 || n_chunks > max_chunks)
    return fail(PA_ERR_INVALID_ARG, "n_chunks must be in [1, %d] (got %d)", max_chunks, n_chunks);
  for (int c = 0; c < n_chunks; ++c) {
    const int rc = host_fwd_checks(q, k_chunks[c], v_chunks[c], o, lse, B, H, Nq, nk_chunks[c], d, scale);
    if (rc != PA_OK) return rc;
  }
  if (Nq == 0) return PA_OK;
  constexpr int kMax = 3 + 2 * 64;
  const void* ptrs[kMax];
  const char* names[kMax];
  int n = 0;
  ptrs[n] = q, names[n++] = "q";
  ptrs[n] = o, names[n++] = "o";
  ptrs[n] = lse, names[n++] = "lse";
  for (int c = 0; c < n_chunks && n + 2 <= kMax; ++c) {
    ptrs[n] = k_chunks[c], names[n++] = "k chunk";
    ptrs[n] = v_chunks[c], names[n++] = "v chunk";
  }
  return device_checks(ptrs, names, n, st);
}

}  // namespace

extern "C" {

int pa_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq,
                int Nk, int d, float scale, void* stream) {
  g_err[0] = '\0';
  DeviceState* st = nullptr;
  int rc = check_fwd_args(q, k, v, o, lse, B, H, Nq, Nk, d, scale, &st);
  if (rc != PA_OK || st == nullptr) return rc;
  return launch_bf16(st, d, q, &k, &v, &Nk, 1, o, lse, B * H, Nq, scale, static_cast<cudaStream_t>(stream));
}

int pa_attn_fwd_accum(const void* q, const void* k, const void* v, float* o_acc, float* lse_acc, void* o, int B,
                      int H, int Nq, int Nk, int d, float scale, int flags, void* stream) {
  g_err[0] = '\0';
  if (flags & ~(PA_ACCUM_FIRST | PA_ACCUM_FINAL)) return fail(PA_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  const bool final_fold = (flags & PA_ACCUM_FINAL) != 0;
  if (final_fold && !o) return fail(PA_ERR_INVALID_ARG, "PA_ACCUM_FINAL needs the bf16 output o");
  if (!final_fold && o) return fail(PA_ERR_INVALID_ARG, "o is written only with PA_ACCUM_FINAL: pass null");
  int rc = host_fwd_checks(q, k, v, o_acc, lse_acc, B, H, Nq, Nk, d, scale, 2, 4, o);
  if (rc != PA_OK || Nq == 0) return rc;
  const void* ptrs[6] = {q, k, v, o_acc, lse_acc, o ? o : o_acc};
  const char* names[6] = {"q", "k", "v", "o_acc", "lse_acc", "o"};
  DeviceState* st = nullptr;
  if ((rc = device_checks(ptrs, names, 6, &st)) != PA_OK) return rc;
  AccArgs acc;
  acc.acc_o = o_acc;
  acc.acc_lse = lse_acc;
  acc.flags = (flags & PA_ACCUM_FIRST ? pa::kAccFirst : 0) | (final_fold ? pa::kAccFinal : 0);
  return launch_bf16(st, d, q, &k, &v, &Nk, 1, o, nullptr, B * H, Nq, scale, static_cast<cudaStream_t>(stream), acc);
}

int pa_attn_fwd_fp8(const void* q, const void* k, const void* v, float q_scale, float k_scale, float v_scale,
                    void* o, float* lse, int B, int H, int Nq, int Nk, int d, float scale, void* stream) {
  g_err[0] = '\0';
  for (float sc : {q_scale, k_scale, v_scale})
    if (!std::isfinite(sc) || !(sc > 0.f)) return fail(PA_ERR_INVALID_ARG, "dequantisation scales must be finite and > 0");
  DeviceState* st = nullptr;
  int rc = host_fwd_checks(q, k, v, o, lse, B, H, Nq, Nk, d, scale, 1);
  if (rc != PA_OK) return rc;
  if (d != 128) return fail(PA_ERR_UNSUPPORTED, "the e4m3 forward needs d = 128 (got %d)", d);
  rc = check_fwd_args(q, k, v, o, lse, B, H, Nq, Nk, d, scale, &st, 1);
  if (rc != PA_OK || st == nullptr) return rc;
  return launch_fwd<128, true>(st, q, &k, &v, &Nk, 1, o, lse, B * H, Nq, scale, static_cast<cudaStream_t>(stream),
                               q_scale * k_scale, v_scale);
}

int pa_attn_fwd_fp8_dev(const void* q, const void* k, const void* v, const float* q_scale, const float* k_scale,
                        const float* v_scale, void* o, float* lse, int B, int H, int Nq, int Nk, int d, float scale,
                        void* stream) {
  g_err[0] = '\0';
  if (!q_scale || !k_scale || !v_scale) return fail(PA_ERR_INVALID_ARG, "null scale pointer");
  if (!aligned(q_scale, 4) || !aligned(k_scale, 4) || !aligned(v_scale, 4))
    return fail(PA_ERR_MISALIGNED, "scale pointers must be 4-byte aligned");
  DeviceState* st = nullptr;
  int rc = host_fwd_checks(q, k, v, o, lse, B, H, Nq, Nk, d, scale, 1);
  if (rc != PA_OK) return rc;
  if (d != 128) return fail(PA_ERR_UNSUPPORTED, "the e4m3 forward needs d = 128 (got %d)", d);
  rc = check_fwd_args(q, k, v, o, lse, B, H, Nq, Nk, d, scale, &st, 1);
  if (rc != PA_OK || st == nullptr) return rc;
  int dev = 0;
  const float* sp[3] = {q_scale, k_scale, v_scale};
  for (int i = 0; i < 3; ++i)
    if ((rc = check_device_ptr(sp[i], "scale", &dev)) != PA_OK) return rc;
  return launch_fwd<128, true>(st, q, &k, &v, &Nk, 1, o, lse, B * H, Nq, scale, static_cast<cudaStream_t>(stream),
                               1.f, 1.f, sp);
}

int pa_quantize_e4m3(const void* x, long long n, void* q, float* scale, void* stream) {
  g_err[0] = '\0';
  if (!x || !q || !scale) return fail(PA_ERR_INVALID_ARG, "null pointer argument");
  if (n < 1) return fail(PA_ERR_INVALID_ARG, "n must be >= 1 (got %lld)", n);
  if (!aligned(x, 16) || !aligned(q, 16)) return fail(PA_ERR_MISALIGNED, "x and q must be 16-byte aligned");
  if (!aligned(scale, 4)) return fail(PA_ERR_MISALIGNED, "scale must be 4-byte aligned");
  if (overlap(x, static_cast<uint64_t>(n) * 2, q, static_cast<uint64_t>(n)) ||
      overlap(x, static_cast<uint64_t>(n) * 2, scale, 4) || overlap(q, static_cast<uint64_t>(n), scale, 4))
    return fail(PA_ERR_INVALID_ARG, "x, q and scale must not overlap");
  (void)cudaGetLastError();
  int dev = 0, rc;
  const void* ptrs[3] = {x, q, scale};
  const char* names[3] = {"x", "q", "scale"};
  for (int i = 0; i < 3; ++i)
    if ((rc = check_device_ptr(ptrs[i], names[i], &dev)) != PA_OK) return rc;
  DeviceState* st = nullptr;
  if ((rc = device_state(dev, &st)) != PA_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned* word = reinterpret_cast<unsigned*>(scale);
  cudaError_t e = cudaMemsetAsync(word, 0, 4, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  const long long n8 = n / 8;
  const long long want = (n8 + pa::quant::kThreads - 1) / pa::quant::kThreads;
  const int grid = static_cast<int>(std::max(1LL, std::min(want, 8LL * st->sm_count)));
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  pa::quant::amax_kernel<<<grid, pa::quant::kThreads, 0, s>>>(xb, n, word);
  pa::quant::quantize_kernel<<<grid, pa::quant::kThreads, 0, s>>>(xb, n, word, static_cast<uint8_t*>(q));
  pa::quant::scale_kernel<<<1, 1, 0, s>>>(word, st->status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  return PA_OK;
}

int pa_attn_fwd_chunks(const void* q, const void* const* k_chunks, const void* const* v_chunks,
                       const int* nk_chunks, int n_chunks, void* o, float* lse, int B, int H, int Nq, int d,
                       float scale, void* stream) {
  g_err[0] = '\0';
  DeviceState* st = nullptr;
  const int rc = check_chunk_args(q, k_chunks, v_chunks, nk_chunks, n_chunks, pa::single::kMaxChunks, o, lse, B, H,
                                  Nq, d, scale, &st);
  if (rc != PA_OK || st == nullptr) return rc;
  return launch_bf16(st, d, q, k_chunks, v_chunks, nk_chunks, n_chunks, o, lse, B * H, Nq, scale,
                     static_cast<cudaStream_t>(stream));
}

int pa_attn_merge(const void* o_parts, const float* lse_parts, int n_parts, void* o, float* lse, int B, int H,
                  int N, int d, void* stream) {
  g_err[0] = '\0';
  if (!o_parts || !lse_parts || !o || !lse) return fail(PA_ERR_INVALID_ARG, "null pointer argument");
  if (n_parts < 1) return fail(PA_ERR_INVALID_ARG, "n_parts must be >= 1 (got %d)", n_parts);
  if (B < 1 || H < 1) return fail(PA_ERR_INVALID_ARG, "B and H must be >= 1 (got %d, %d)", B, H);
  if (N < 0) return fail(PA_ERR_INVALID_ARG, "N must be >= 0 (got %d)", N);
  if (d != 64 && d != 128) return fail(PA_ERR_UNSUPPORTED, "d must be 64 or 128 (got %d)", d);
  if (!aligned(o_parts, 16) || !aligned(o, 16))
    return fail(PA_ERR_MISALIGNED, "o_parts and o must be 16-byte aligned");
  if (!aligned(lse_parts, 4) || !aligned(lse, 4))
    return fail(PA_ERR_MISALIGNED, "lse_parts and lse must be 4-byte aligned");
  if (N == 0) return PA_OK;
  const long long rows = static_cast<long long>(B) * H * N;
  const uint64_t obytes = static_cast<uint64_t>(rows) * d * 2;
  const uint64_t lbytes = static_cast<uint64_t>(rows) * 4;
  if (overlap(o_parts, obytes * n_parts, o, obytes) || overlap(o_parts, obytes * n_parts, lse, lbytes) ||
      overlap(lse_parts, lbytes * n_parts, o, obytes) || overlap(lse_parts, lbytes * n_parts, lse, lbytes) ||
      overlap(o, obytes, lse, lbytes))
    return fail(PA_ERR_INVALID_ARG, "outputs overlap an input");

  (void)cudaGetLastError();
  int dev = 0, rc;
  const void* ptrs[4] = {o_parts, lse_parts, o, lse};
  const char* names[4] = {"o_parts", "lse_parts", "o", "lse"};
  for (int i = 0; i < 4; ++i)
    if ((rc = check_device_ptr(ptrs[i], names[i], &dev)) != PA_OK) return rc;
  DeviceState* st = nullptr;
  if ((rc = device_state(dev, &st)) != PA_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 64) return launch_merge<64>(st, o_parts, lse_parts, n_parts, o, lse, rows, s);
  return launch_merge<128>(st, o_parts, lse_parts, n_parts, o, lse, rows, s);
}

int pa_residual_diff(const void* cur, const void* prev, long long n, float* out, void* stream) {
  g_err[0] = '\0';
  if (!cur || !prev || !out) return fail(PA_ERR_INVALID_ARG, "null pointer argument");
  if (n < 1) return fail(PA_ERR_INVALID_ARG, "n must be >= 1 (got %lld)", n);
  if (!aligned(cur, 16) || !aligned(prev, 16)) return fail(PA_ERR_MISALIGNED, "cur and prev must be 16-byte aligned");
  if (!aligned(out, 4)) return fail(PA_ERR_MISALIGNED, "out must be 4-byte aligned");
  const uint64_t bytes = static_cast<uint64_t>(n) * 2;
  if (overlap(cur, bytes, out, 4) || overlap(prev, bytes, out, 4))
    return fail(PA_ERR_INVALID_ARG, "out overlaps an input");
  (void)cudaGetLastError();
  int dev = 0, rc;
  const void* ptrs[3] = {cur, prev, out};
  const char* names[3] = {"cur", "prev", "out"};
  for (int i = 0; i < 3; ++i)
    if ((rc = check_device_ptr(ptrs[i], names[i], &dev)) != PA_OK) return rc;
  DeviceState* st = nullptr;
  if ((rc = device_state(dev, &st)) != PA_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // A fixed grid for a given size and device (the result's rounding does not
  // depend on scheduling): enough blocks to keep every SM streaming.
  const long long vecs = (n / 8 + pa::kRdThreads - 1) / pa::kRdThreads;
  const int grid = static_cast<int>(std::max<long long>(
      1, std::min<long long>(vecs, std::min<long long>(4LL * st->sm_count, pa::kRdMaxBlocks))));
  pa::residual_diff_partial_kernel<<<grid, pa::kRdThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(cur),
                                                                   static_cast<const __nv_bfloat16*>(prev), n);
  pa::residual_diff_final_kernel<<<1, pa::kRdThreads, 0, s>>>(grid, out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "residual_diff launch");
  return PA_OK;
}

int pa_attn_chunks_noalloc(const void* q, const void* const* k_chunks, const void* const* v_chunks,
                           const int* nk_chunks, int n_chunks, void* o, float* lse, int B, int H, int Nq, int d,
                           float scale, void* stream) {
  g_err[0] = '\0';
  if (!q || !k_chunks || !v_chunks || !nk_chunks || !o || !lse)
    return fail(PA_ERR_INVALID_ARG, "null pointer argument");
  if (n_chunks < 1 || n_chunks > pa::kNoAllocMaxChunks)
    return fail(PA_ERR_INVALID_ARG, "n_chunks must be in [1, %d] (got %d)", pa::kNoAllocMaxChunks, n_chunks);
  if (B < 1 || H < 1 || Nq < 0) return fail(PA_ERR_INVALID_ARG, "B, H must be >= 1 and Nq >= 0");
  if (d != 64 && d != 128) return fail(PA_ERR_UNSUPPORTED, "d must be 64 or 128 (got %d)", d);
  // Partials: n blocks of [B*H, Nq, d] bf16, then n blocks of [B*H, Nq] fp32.
  const unsigned long long rows = static_cast<unsigned long long>(B) * H * Nq;
  const unsigned long long o_part = rows * d * 2;
  const unsigned long long lse_off = ((o_part * n_chunks) + 255ull) & ~255ull;
  const unsigned long long need = (n_chunks > 1) ? lse_off + rows * 4ull * n_chunks : 0ull;
  if (need > pa::kNoAllocScratchBytes)
    return fail(PA_ERR_INVALID_ARG, "the %d partial results need %llu bytes of scratch; the limit is %llu", n_chunks,
                need, pa::kNoAllocScratchBytes);
  DeviceState* st = nullptr;
  const int rc0 = check_chunk_args(q, k_chunks, v_chunks, nk_chunks, n_chunks, pa::kNoAllocMaxChunks, o, lse, B, H,
                                   Nq, d, scale, &st);
  if (rc0 != PA_OK || st == nullptr) return rc0;  // st is null when Nq == 0
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int bh = B * H;
  auto fwd = [&](const void* k, const void* v, void* out, float* out_lse, int nk) {
    return launch_bf16(st, d, q, &k, &v, &nk, 1, out, out_lse, bh, Nq, scale, s);
  };
  if (n_chunks == 1) return fwd(k_chunks[0], v_chunks[0], o, lse, nk_chunks[0]);
  // Every forward below writes its whole partial block before the merge reads
  // it, so nothing left in the shared array by an earlier call is ever read.
  unsigned char* scratch = st->noalloc_scratch;
  float* lse_parts = reinterpret_cast<float*>(scratch + lse_off);
  for (int c = 0; c < n_chunks; ++c) {
    const int rc = fwd(k_chunks[c], v_chunks[c], scratch + o_part * c, lse_parts + rows * c, nk_chunks[c]);
    if (rc != PA_OK) return rc;
  }
  return d == 64 ? launch_merge<64>(st, scratch, lse_parts, n_chunks, o, lse, static_cast<long long>(rows), s)
                 : launch_merge<128>(st, scratch, lse_parts, n_chunks, o, lse, static_cast<long long>(rows), s);
}

const char* pa_status_string(int code) {
  switch (code) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG: invalid argument";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED: unsupported shape or device";
    case PA_ERR_MISALIGNED: return "PA_ERR_MISALIGNED: pointer alignment";
    case PA_ERR_CUDA: return "PA_ERR_CUDA: CUDA runtime or driver error";
    case PA_ERR_TIMEOUT: return "PA_ERR_TIMEOUT: a device-side bounded wait gave up";
    case PA_ERR_BAD_INPUT: return "PA_ERR_BAD_INPUT: a value read on the device was not finite or not positive";
    default: return "unknown status code";
  }
}

const char* pa_last_error(void) { return g_err; }

int pa_poll_device_status(void) {
  g_err[0] = '\0';
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  DeviceState* st = nullptr;
  int rc = device_state(dev, &st);
  if (rc != PA_OK) return rc;
  int value = 0;
  e = cudaMemcpy(&value, st->status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
  const int zero = 0;
  e = cudaMemcpy(st->status, &zero, sizeof(int), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the device status word");
  return value;
}

int pa_selftest_timeout(int limit_us, void* stream) {
  g_err[0] = '\0';
  if (limit_us < 1 || limit_us > 1000000) return fail(PA_ERR_INVALID_ARG, "limit_us must be in [1, 1e6]");
  (void)cudaGetLastError();
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  DeviceState* st = nullptr;
  int rc = device_state(dev, &st);
  if (rc != PA_OK) return rc;
  pa::timeout_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(limit_us) * 1000ull, st->status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "timeout probe launch");
  return PA_OK;
}

int pa_set_wait_limit_ms(int ms) {
  g_err[0] = '\0';
  if (ms < 1 || ms > 600000) return fail(PA_ERR_INVALID_ARG, "ms must be in [1, 600000] (got %d)", ms);
  g_wait_limit_ns.store(static_cast<unsigned long long>(ms) * 1000000ull, std::memory_order_relaxed);
  return PA_OK;
}

int pa_version(void) { return 200; }

}  // extern "C"
