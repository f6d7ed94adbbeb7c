// fa_host.cuh — the host side of libfa.so: argument checks, tensor maps,
// launches and the C ABI entry points of include/fa.h (except fa_fwd_host,
// in fa_host_pipeline.cuh). Included once, at the end of fa_fwd_sm100.cu,
// after the kernels it launches.

// ==================================================================== host
namespace {

thread_local char g_err[512] = "";
unsigned long long g_timeout_ns = 4000ull * 1000000ull;

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
using AddressRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);
using CtxGetCurrentFn = CUresult (*)(CUcontext*);

struct DriverFns {
  EncodeTiledFn encode = nullptr;
  AddressRangeFn range = nullptr;
  CtxGetCurrentFn ctx_current = nullptr;
  bool ok = false;
};

const DriverFns& driver_fns() {
  static DriverFns fns;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q1, q2, q3;
    void* f1 = nullptr;
    void* f2 = nullptr;
    void* f3 = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f1, 12000, cudaEnableDefault,
                                         &q1) == cudaSuccess &&
        q1 == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &f2, 12000, cudaEnableDefault,
                                         &q2) == cudaSuccess &&
        q2 == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f3, 12000, cudaEnableDefault,
                                         &q3) == cudaSuccess &&
        q3 == cudaDriverEntryPointSuccess) {
      fns.encode = reinterpret_cast<EncodeTiledFn>(f1);
      fns.range = reinterpret_cast<AddressRangeFn>(f2);
      fns.ctx_current = reinterpret_cast<CtxGetCurrentFn>(f3);
      fns.ok = true;
    }
  });
  return fns;
}

struct DeviceInfo {
  bool init = false;
  bool sm100 = false;
  int sms = 0;
  long long l2_bytes = 0;
  bool attr_set[11] = {};
  bool bwd_attr_set[4] = {false, false, false, false};
};
DeviceInfo g_dev[64];
std::mutex g_dev_mu;

// [ptr, ptr + bytes) must lie inside one device allocation of the current device.
int check_range(const char* name, const void* ptr, size_t bytes, size_t align) {
  if (ptr == nullptr) return fail(FA_ERR_INVALID_ARG, "%s is NULL", name);
  if (reinterpret_cast<uintptr_t>(ptr) % align != 0)
    return fail(FA_ERR_INVALID_ARG, "%s is not %zu-byte aligned", name, align);
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
    cudaGetLastError();
    return fail(FA_ERR_INVALID_ARG, "%s is not a CUDA pointer", name);
  }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
    return fail(FA_ERR_INVALID_ARG, "%s is not device memory", name);
  int dev = -1;
  cudaGetDevice(&dev);
  if (a.device != dev) return fail(FA_ERR_INVALID_ARG, "%s lives on device %d, not %d", name, a.device, dev);
  CUdeviceptr base = 0;
  size_t size = 0;
  if (driver_fns().range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS)
    return fail(FA_ERR_INVALID_ARG, "%s: no allocation found", name);
  const uintptr_t p = reinterpret_cast<uintptr_t>(ptr);
  if (p + bytes > static_cast<uintptr_t>(base) + size)
    return fail(FA_ERR_INVALID_ARG, "%s: %zu bytes run past its allocation", name, bytes);
  return FA_OK;
}

// Dense 3-D map [dims[2]][dims[1]][dims[0]] of `elem`-byte elements.
int encode_map(CUtensorMap* map, const void* ptr, CUtensorMapDataType type, int elem,
               const cuuint64_t (&dims)[3], int box_cols, int box_rows, CUtensorMapSwizzle swz) {
  const cuuint64_t strides[2] = {dims[0] * elem, dims[0] * elem * dims[1]};
  const cuuint32_t box[3] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = driver_fns().encode(map, type, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return FA_OK;
}

int make_map(CUtensorMap* map, const void* ptr, bool bf16, int d, int n, long long heads,
             int box_cols, int box_rows, CUtensorMapSwizzle swz) {
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)n, (cuuint64_t)heads};
  return encode_map(map, ptr, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                    2, dims, box_cols, box_rows, swz);
}

// 3-D map of bytes [heads][rows][inner] with 128×128-byte boxes, 128-byte swizzle.
int make_map_u8(CUtensorMap* map, const void* ptr, int inner, int rows, long long heads) {
  const cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)heads};
  return encode_map(map, ptr, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, dims, 128, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int D, bool BF16, int MODE = 0>
int launch(const void* q, const void* k, const void* v, void* o, const fa::Params& prm,
           cudaStream_t stream, DeviceInfo& info, int slot, float* final_lse,
           const void* bias = nullptr, long long bias_planes = 0) {
  using L = fa::Layout<D, MODE>;
  auto kern = fa::fa_fwd_kernel<D, BF16, MODE>;
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!info.attr_set[slot]) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC) !=
          cudaSuccess)
        return fail(FA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(cudaGetLastError()));
      cudaFuncAttributes fa_attr;
      if (cudaFuncGetAttributes(&fa_attr, kern) != cudaSuccess)
        return fail(FA_ERR_CUDA, "cudaFuncGetAttributes: %s", cudaGetErrorString(cudaGetLastError()));
      // The setmaxnreg split (2×176 + 80 + 80 per 128 threads) needs exactly 128
      // registers per thread at launch; anything else could never be satisfied.
      if (fa_attr.numRegs != 128)
        return fail(FA_ERR_UNSUPPORTED, "kernel built with %d registers per thread, need 128",
                    fa_attr.numRegs);
      info.attr_set[slot] = true;
    }
  }
  CUtensorMap tq, tk, tv, to;
  const fa::Shape& s = prm.s;
  int rc;
  if (MODE == 2) {
    // E4M3 bytes: Q, K [heads][N][D] in 128×128-byte boxes; v is the transposed
    // copy Vᵀ [heads][D][N] (row stride N bytes, a multiple of 16)
    if ((rc = make_map_u8(&tq, q, D, s.N, (long long)s.B * s.Hq)) != FA_OK) return rc;
    if ((rc = make_map_u8(&tk, k, D, s.N, (long long)s.B * s.Hk)) != FA_OK) return rc;
    if ((rc = make_map_u8(&tv, v, s.N, D, (long long)s.B * s.Hk)) != FA_OK) return rc;
  } else {
    if ((rc = make_map(&tq, q, BF16, D, s.N, (long long)s.B * s.Hq, 64, fa::BM,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK) return rc;
    if ((rc = make_map(&tk, k, BF16, D, s.N, (long long)s.B * s.Hk, 64, fa::BN,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK) return rc;
    if ((rc = make_map(&tv, v, BF16, D, s.N, (long long)s.B * s.Hk, 64, fa::BN,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK) return rc;
  }
  if ((rc = make_map(&to, o, BF16, D, s.N, (long long)s.B * s.Hq, 32, 32,
                     CU_TENSOR_MAP_SWIZZLE_64B)) != FA_OK) return rc;
  CUtensorMap tb;
  memset(&tb, 0, sizeof(tb));
  // bias planes [planes][N][N]: boxes of 64 keys × 128 query rows
  if (MODE == 1 && (rc = make_map(&tb, bias, BF16, s.N, s.N, bias_planes, 64, fa::BM,
                             CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK) return rc;
  const int grid = s.num_units < info.sms ? s.num_units : info.sms;
  kern<<<grid, fa::NUM_THREADS, L::ALLOC, stream>>>(tq, tk, tv, to, tb, prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "launch failed: %s", cudaGetErrorString(e));
  if (prm.o_part != nullptr) {
    const long long rows = (long long)s.B * s.Hq * s.N;
    long long blocks = (rows + 7) / 8;
    if (blocks > (long long)info.sms * 16) blocks = (long long)info.sms * 16;
    fa::fa_merge_splits_kernel<D, BF16><<<(unsigned)blocks, 256, 0, stream>>>(
        prm.o_part, prm.lse_part, s.splits, rows, o, final_lse);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(FA_ERR_CUDA, "merge launch failed: %s", cudaGetErrorString(e));
  }
  return FA_OK;
}

// Workspace of a split-KV call: partial O then partial LSE, fp32.
size_t splitkv_bytes(long long heads_q, int N, int d, int splits) {
  const size_t rows = (size_t)heads_q * N * (size_t)splits;
  const size_t o_bytes = (rows * d * 4 + 255) / 256 * 256;
  return o_bytes + (rows * 4 + 255) / 256 * 256;
}

}  // namespace

extern "C" {

int fa_version(void) { return 100; }

const char* fa_last_error_string(void) { return g_err; }

int fa_set_wait_timeout_ms(int ms) {
  if (ms < 1 || ms > 600000) return fail(FA_ERR_INVALID_ARG, "timeout %d ms out of [1, 600000]", ms);
  g_timeout_ns = (unsigned long long)ms * 1000000ull;
  return FA_OK;
}

int fa_num_units(int B, int Hq, int Hk, int N, int causal) {
  if (B < 1 || Hq < 1 || Hk < 1 || N < 1 || Hq % Hk != 0)
    return fail(FA_ERR_INVALID_ARG, "bad shape");
  const long long units = (long long)B * Hk * ((((long long)Hq / Hk) * ((N + 127) / 128) + 1) / 2);
  if (units > 0x7fffffffLL) return fail(FA_ERR_INVALID_ARG, "too many work units");
  return fa::make_shape(B, Hq, Hk, N, causal).num_units;
}

int fa_unit_info(int B, int Hq, int Hk, int N, int causal, int u, int32_t* out) {
  const int nu = fa_num_units(B, Hq, Hk, N, causal);
  if (nu < 0) return nu;
  if (out == nullptr || u < 0 || u >= nu) return fail(FA_ERR_INVALID_ARG, "bad unit index");
  fa::Unit U;
  fa::decode_unit(fa::make_shape(B, Hq, Hk, N, causal), u, U);
  const int32_t vals[8] = {U.b, U.hk, U.hq[0], U.mb[0], U.present[0], U.hq[1], U.mb[1], U.present[1]};
  memcpy(out, vals, sizeof(vals));
  return FA_OK;
}

int fa_unit_kv_range(int B, int Hq, int Hk, int N, int causal, int num_splits, int u,
                     int key_len, int32_t* out) {
  const int nu = fa_num_units(B, Hq, Hk, N, causal);
  if (nu < 0) return nu;
  if (num_splits < 1 || num_splits > 16) return fail(FA_ERR_INVALID_ARG, "num_splits out of [1, 16]");
  if (out == nullptr || u < 0 || (long long)u >= (long long)nu * num_splits)
    return fail(FA_ERR_INVALID_ARG, "bad unit index");
  if (key_len < 0 || key_len > N) return fail(FA_ERR_INVALID_ARG, "key_len out of [0, N]");
  const fa::Shape s = fa::make_shape(B, Hq, Hk, N, causal, num_splits);
  fa::Unit U;
  fa::decode_unit(s, u, U);
  fa::resolve_unit(s, key_len, U);
  const int32_t vals[12] = {U.b, U.hk, U.hq[0], U.mb[0], U.present[0], U.hq[1], U.mb[1],
                            U.present[1], U.split, U.j0, U.n[0], U.n[1]};
  memcpy(out, vals, sizeof(vals));
  return FA_OK;
}

int fa_unit_for(int cta, int it, int grid) { return fa::unit_for(cta, it, grid); }

int fa_unit_for_grouped(int B, int Hq, int Hk, int N, int causal, int num_splits, int groups,
                        int cta, int it, int grid) {
  const int nu = fa_num_units(B, Hq, Hk, N, causal);
  if (nu < 0) return nu;
  if (num_splits < 1 || num_splits > 16) return fail(FA_ERR_INVALID_ARG, "num_splits out of [1, 16]");
  if (groups < 2 || groups > B * Hk || !causal)
    return fail(FA_ERR_INVALID_ARG, "groups out of [2, B·Hk], or not causal");
  if (grid < 1 || cta < 0 || cta >= grid || it < 0) return fail(FA_ERR_INVALID_ARG, "bad CTA or iteration");
  fa::Shape s = fa::make_shape(B, Hq, Hk, N, causal, num_splits, groups);
  fa::set_group_grid(s, grid);
  return fa::unit_for_grouped(s, cta, it, grid);
}

int fa_unit_groups(int B, int Hq, int Hk, int N, int d, int causal, int grid, long long l2_bytes) {
  if (B < 1 || Hq < 1 || Hk < 1 || N < 1 || Hq % Hk != 0 || grid < 1 || d < 1 || l2_bytes < 0)
    return fail(FA_ERR_INVALID_ARG, "bad arguments");
  return fa::group_count(B, Hq, Hk, N, causal, grid, 4LL * N * d, l2_bytes);
}

int fa_unit_kv_range_grouped(int B, int Hq, int Hk, int N, int causal, int num_splits, int groups,
                             int u, int key_len, int32_t* out) {
  const int nu = fa_num_units(B, Hq, Hk, N, causal);
  if (nu < 0) return nu;
  if (num_splits < 1 || num_splits > 16) return fail(FA_ERR_INVALID_ARG, "num_splits out of [1, 16]");
  if (groups < 0 || groups > B * Hk) return fail(FA_ERR_INVALID_ARG, "groups out of [0, B·Hk]");
  if (out == nullptr || u < 0 || (long long)u >= (long long)nu * num_splits)
    return fail(FA_ERR_INVALID_ARG, "bad unit index");
  if (key_len < 0 || key_len > N) return fail(FA_ERR_INVALID_ARG, "key_len out of [0, N]");
  const fa::Shape s = fa::make_shape(B, Hq, Hk, N, causal, num_splits, groups);
  fa::Unit U;
  fa::decode_unit(s, u, U);
  fa::resolve_unit(s, key_len, U);
  const int32_t vals[12] = {U.b, U.hk, U.hq[0], U.mb[0], U.present[0], U.hq[1], U.mb[1],
                            U.present[1], U.split, U.j0, U.n[0], U.n[1]};
  memcpy(out, vals, sizeof(vals));
  return FA_OK;
}

}  // extern "C"

// ============================================ split-KV with a static scratch
// The scratch of fa_fwd_splitkv_static: a file-scope device array, so the
// call allocates nothing. It exists once per device that loads this module
// and is shared by every call on that device.
static __device__ __align__(256) uint8_t g_fa_static_scratch[FA_STATIC_SCRATCH_BYTES];

namespace {
// Device address of g_fa_static_scratch per device, with the context it was
// looked up in: a new primary context (after cudaDeviceReset) reloads the
// module, so the address is looked up again when the current context differs.
struct ScratchAddr {
  CUcontext ctx = nullptr;
  void* ptr = nullptr;
};
ScratchAddr g_scratch[64];

int static_scratch(int dev, void** ptr) {
  CUcontext ctx = nullptr;
  if (driver_fns().ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
    return fail(FA_ERR_CUDA, "no current CUDA context");
  std::lock_guard<std::mutex> lk(g_dev_mu);
  ScratchAddr& a = g_scratch[dev];
  if (a.ptr == nullptr || a.ctx != ctx) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_fa_static_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(FA_ERR_CUDA, "cudaGetSymbolAddress of the static scratch: %s",
                  cudaGetErrorString(e));
    a.ctx = ctx;
    a.ptr = p;
  }
  *ptr = a.ptr;
  return FA_OK;
}
}  // namespace

namespace {
int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hk,
             int N, int d, float scale, int causal, const int32_t* key_pad_lens, int splits,
             void* workspace, size_t workspace_bytes, void* stream, int dtype,
             const void* bias = nullptr, int bias_B = 0, int bias_H = 0,
             bool library_scratch = false) {
  g_err[0] = '\0';
  // ---- arguments that need no CUDA call
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr)
    return fail(FA_ERR_INVALID_ARG, "q, k, v and o must be non-NULL");
  if (B < 1 || Hq < 1 || Hk < 1 || N < 1)
    return fail(FA_ERR_INVALID_ARG, "B, Hq, Hk and N must be >= 1");
  if (Hq % Hk != 0) return fail(FA_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hk (%d)", Hq, Hk);
  if (d != 64 && d != 128)
    return fail(FA_ERR_UNSUPPORTED, "head dim %d not supported (64 or 128)", d);
  if (dtype != FA_FP16 && dtype != FA_BF16) return fail(FA_ERR_UNSUPPORTED, "unknown dtype %d", dtype);
  if (!std::isfinite(scale)) return fail(FA_ERR_INVALID_ARG, "scale must be finite");
  if (causal != 0 && causal != 1) return fail(FA_ERR_INVALID_ARG, "causal must be 0 or 1");
  const long long heads_q = (long long)B * Hq, heads_k = (long long)B * Hk;
  if (heads_q > 0x7fffffffLL || N > (1 << 30))
    return fail(FA_ERR_INVALID_ARG, "problem too large for 32-bit tile coordinates");
  if (fa_num_units(B, Hq, Hk, N, causal) < 0) return FA_ERR_INVALID_ARG;
  if (splits < 1 || splits > 16) return fail(FA_ERR_INVALID_ARG, "num_splits %d out of [1, 16]", splits);
  if ((long long)fa_num_units(B, Hq, Hk, N, causal) * splits > 0x7fffffffLL)
    return fail(FA_ERR_INVALID_ARG, "too many work units");
  const size_t bias_bytes = bias ? (size_t)bias_B * bias_H * N * (size_t)N * 2 : 0;
  if (bias != nullptr) {
    if (bias_B != 1 && bias_B != B)
      return fail(FA_ERR_INVALID_ARG, "bias batch dimension %d must be 1 or B (%d)", bias_B, B);
    if (bias_H != 1 && bias_H != Hq)
      return fail(FA_ERR_INVALID_ARG, "bias head dimension %d must be 1 or Hq (%d)", bias_H, Hq);
    if (N % 8 != 0)
      return fail(FA_ERR_UNSUPPORTED, "bias needs N %% 8 == 0 (16-byte rows), N = %d", N);
    if (splits != 1) return fail(FA_ERR_UNSUPPORTED, "bias with split-KV is not supported");
  }
  // ---- device and buffers
  if (!driver_fns().ok) return fail(FA_ERR_CUDA, "CUDA driver entry points unavailable");
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return fail(FA_ERR_CUDA, "no current CUDA device");
  DeviceInfo& info = g_dev[dev];
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!info.init) {
      cudaDeviceProp prop;
      if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess)
        return fail(FA_ERR_CUDA, "cudaGetDeviceProperties failed");
      info.sm100 = prop.major == 10 && prop.minor == 0;
      info.sms = prop.multiProcessorCount;
      info.l2_bytes = prop.l2CacheSize;
      info.init = true;
    }
  }
  if (!info.sm100) return fail(FA_ERR_UNSUPPORTED, "device %d is not sm_100", dev);
  const size_t q_bytes = (size_t)heads_q * N * d * 2, kv_bytes = (size_t)heads_k * N * d * 2;
  int rc;
  if ((rc = check_range("q", q, q_bytes, 16)) != FA_OK) return rc;
  if ((rc = check_range("k", k, kv_bytes, 16)) != FA_OK) return rc;
  if ((rc = check_range("v", v, kv_bytes, 16)) != FA_OK) return rc;
  if ((rc = check_range("o", o, q_bytes, 16)) != FA_OK) return rc;
  if (lse != nullptr && (rc = check_range("lse", lse, (size_t)heads_q * N * 4, 4)) != FA_OK) return rc;
  if (key_pad_lens != nullptr &&
      (rc = check_range("key_pad_lens", key_pad_lens, (size_t)B * 4, 4)) != FA_OK)
    return rc;
  const uintptr_t ob = reinterpret_cast<uintptr_t>(o), oe = ob + q_bytes;
  auto overlaps = [&](const void* x, size_t n) {
    const uintptr_t xb = reinterpret_cast<uintptr_t>(x);
    return xb < oe && ob < xb + n;
  };
  if (overlaps(q, q_bytes) || overlaps(k, kv_bytes) || overlaps(v, kv_bytes) ||
      (lse != nullptr && overlaps(lse, (size_t)heads_q * N * 4)))
    return fail(FA_ERR_INVALID_ARG, "o overlaps an input or lse");
  if (bias != nullptr) {
    if ((rc = check_range("bias", bias, bias_bytes, 16)) != FA_OK) return rc;
    if (overlaps(bias, bias_bytes)) return fail(FA_ERR_INVALID_ARG, "o overlaps bias");
    const uintptr_t bb = reinterpret_cast<uintptr_t>(bias), be = bb + bias_bytes;
    const uintptr_t lb = reinterpret_cast<uintptr_t>(lse);
    if (lse != nullptr && lb < be && bb < lb + (size_t)heads_q * N * 4)
      return fail(FA_ERR_INVALID_ARG, "lse overlaps bias");
  }

  fa::Params prm;
  prm.key_pad_lens = key_pad_lens;
  prm.lse = lse;
  prm.o_part = nullptr;
  prm.lse_part = nullptr;
  prm.o_scale = 1.f;
  prm.bias_bmul = bias_B > 1 ? 1 : 0;
  prm.bias_hmul = bias_H > 1 ? 1 : 0;
  prm.bias_H = bias_H > 0 ? bias_H : 1;
  if (splits > 1) {
    const size_t need = splitkv_bytes(heads_q, N, d, splits);
    if (library_scratch) {
      // fa_fwd_splitkv_static: the library's own scratch, after every other check
      if (need > FA_STATIC_SCRATCH_BYTES)
        return fail(FA_ERR_INVALID_ARG,
                    "split-KV scratch of %zu bytes needed, the static scratch holds %zu; "
                    "use fa_fwd_splitkv with a caller workspace",
                    need, (size_t)FA_STATIC_SCRATCH_BYTES);
      if ((rc = static_scratch(dev, &workspace)) != FA_OK) return rc;
      workspace_bytes = FA_STATIC_SCRATCH_BYTES;
    }
    if (workspace_bytes < need)
      return fail(FA_ERR_INVALID_ARG, "workspace of %zu bytes, need %zu", workspace_bytes, need);
    // The library's own scratch is a module variable, not an allocation the
    // range query knows; its size is checked above.
    if (!library_scratch && (rc = check_range("workspace", workspace, need, 256)) != FA_OK) return rc;
    const uintptr_t wb = reinterpret_cast<uintptr_t>(workspace), we = wb + need;
    auto hits = [&](const void* x, size_t n) {
      const uintptr_t xb = reinterpret_cast<uintptr_t>(x);
      return x != nullptr && xb < we && wb < xb + n;
    };
    if (hits(q, q_bytes) || hits(k, kv_bytes) || hits(v, kv_bytes) || hits(o, q_bytes) ||
        hits(lse, (size_t)heads_q * N * 4) || hits(key_pad_lens, (size_t)B * 4))
      return fail(FA_ERR_INVALID_ARG, "workspace overlaps an argument");
    const size_t rows = (size_t)heads_q * N * splits;
    prm.o_part = reinterpret_cast<float*>(workspace);
    prm.lse_part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) +
                                            (rows * d * 4 + 255) / 256 * 256);
  }
  {
    // head-grouped unit order (a kernel of its own: d = 128, no bias)
    const fa::Shape s0 = fa::make_shape(B, Hq, Hk, N, causal, splits);
    const int grid = s0.num_units < info.sms ? s0.num_units : info.sms;
    const int ng = (d == 128 && bias == nullptr)
                       ? fa::group_count(B, Hq, Hk, N, causal, grid, 4LL * N * d, info.l2_bytes)
                       : 0;
    prm.s = fa::make_shape(B, Hq, Hk, N, causal, splits, ng);
    fa::set_group_grid(prm.s, grid);
  }
  prm.scale_log2 = (float)((double)scale * 1.4426950408889634);
  prm.timeout_ns = g_timeout_ns;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf16 = dtype == FA_BF16;
  if (bias != nullptr) {
    const long long planes = (long long)bias_B * bias_H;
    if (d == 128)
      return bf16 ? launch<128, true, 1>(q, k, v, o, prm, st, info, 4, lse, bias, planes)
                  : launch<128, false, 1>(q, k, v, o, prm, st, info, 5, lse, bias, planes);
    return bf16 ? launch<64, true, 1>(q, k, v, o, prm, st, info, 6, lse, bias, planes)
                : launch<64, false, 1>(q, k, v, o, prm, st, info, 7, lse, bias, planes);
  }
  if (d == 128 && prm.s.ng > 0)
    return bf16 ? launch<128, true, 3>(q, k, v, o, prm, st, info, 9, lse)
                : launch<128, false, 3>(q, k, v, o, prm, st, info, 10, lse);
  if (d == 128)
    return bf16 ? launch<128, true>(q, k, v, o, prm, st, info, 0, lse)
                : launch<128, false>(q, k, v, o, prm, st, info, 1, lse);
  return bf16 ? launch<64, true>(q, k, v, o, prm, st, info, 2, lse)
              : launch<64, false>(q, k, v, o, prm, st, info, 3, lse);
}
}  // namespace

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hk,
           int N, int d, float scale, int causal, const int32_t* key_pad_lens, void* stream,
           int dtype) {
  return fwd_impl(q, k, v, o, lse, B, Hq, Hk, N, d, scale, causal, key_pad_lens, 1, nullptr, 0,
                  stream, dtype);
}

int fa_fwd_bias(const void* q, const void* k, const void* v, const void* bias, int bias_B,
                int bias_H, void* o, float* lse, int B, int Hq, int Hk, int N, int d, float scale,
                int causal, const int32_t* key_pad_lens, void* stream, int dtype) {
  if (bias == nullptr) return fail(FA_ERR_INVALID_ARG, "bias is NULL (use fa_fwd)");
  return fwd_impl(q, k, v, o, lse, B, Hq, Hk, N, d, scale, causal, key_pad_lens, 1, nullptr, 0,
                  stream, dtype, bias, bias_B, bias_H);
}

size_t fa_splitkv_workspace_bytes(int B, int Hq, int N, int d, int num_splits) {
  if (B < 1 || Hq < 1 || N < 1 || (d != 64 && d != 128) || num_splits < 1 || num_splits > 16)
    return 0;
  if (num_splits == 1) return 0;
  return splitkv_bytes((long long)B * Hq, N, d, num_splits);
}

int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                   int Hk, int N, int d, float scale, int causal, const int32_t* key_pad_lens,
                   int num_splits, void* workspace, size_t workspace_bytes, void* stream,
                   int dtype) {
  return fwd_impl(q, k, v, o, lse, B, Hq, Hk, N, d, scale, causal, key_pad_lens, num_splits,
                  workspace, workspace_bytes, stream, dtype);
}



int fa_get_device_status(void) {
  if (cudaDeviceSynchronize() != cudaSuccess)
    return fail(FA_ERR_CUDA, "cudaDeviceSynchronize: %s", cudaGetErrorString(cudaGetLastError()));
  int status = 0;
  if (cudaMemcpyFromSymbol(&status, fa::g_fa_status, sizeof(int)) != cudaSuccess)
    return fail(FA_ERR_CUDA, "reading the status word failed");
  const int zero = 0;
  if (cudaMemcpyToSymbol(fa::g_fa_status, &zero, sizeof(int)) != cudaSuccess)
    return fail(FA_ERR_CUDA, "clearing the status word failed");
  return status;
}

// Runs the bounded wait on a barrier that nothing arrives at, with a limit of
// `ms` milliseconds; returns FA_OK when the wait gave up as designed (and
// leaves FA_ERR_DEVICE_TIMEOUT in the status word).
int fa_selftest_wait_timeout(int ms) {
  if (ms < 1 || ms > 10000) return fail(FA_ERR_INVALID_ARG, "ms out of [1, 10000]");
  int* d_out = nullptr;
  if (cudaMalloc(&d_out, 2 * sizeof(int)) != cudaSuccess) return fail(FA_ERR_CUDA, "cudaMalloc");
  fa::fa_wait_selftest_kernel<<<1, 32>>>((unsigned long long)ms * 1000000ull, d_out);
  int h[2] = {-1, -1};
  cudaError_t e = cudaMemcpy(h, d_out, sizeof(h), cudaMemcpyDeviceToHost);
  cudaFree(d_out);
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "self test: %s", cudaGetErrorString(e));
  if (h[0] != 0 || h[1] != 1) return fail(FA_ERR_CUDA, "self test: wait did not give up");
  return FA_OK;
}

}  // extern "C"


extern "C" int fa_fwd_splitkv_static(const void* q, const void* k, const void* v, void* o,
                                     float* lse, int B, int Hq, int Hk, int N, int d, float scale,
                                     int causal, const int32_t* key_pad_lens, int num_splits,
                                     void* stream, int dtype) {
  return fwd_impl(q, k, v, o, lse, B, Hq, Hk, N, d, scale, causal, key_pad_lens, num_splits,
                  nullptr, 0, stream, dtype, nullptr, 0, 0, /*library_scratch=*/true);
}

// ================================================================ backward
namespace {
struct BwdWs {
  size_t dq_off, lse2_off, dsum_off, bytes;
};
BwdWs bwd_ws(long long heads_q, int N, int d) {
  const size_t npad = (size_t)(N + 127) / 128 * 128;
  BwdWs w;
  w.dq_off = 0;
  w.lse2_off = ((size_t)heads_q * N * d * 4 + 255) / 256 * 256;
  w.dsum_off = w.lse2_off + ((size_t)heads_q * npad * 4 + 255) / 256 * 256;
  w.bytes = w.dsum_off + ((size_t)heads_q * npad * 4 + 255) / 256 * 256;
  return w;
}

template <int D, bool BF16>
int bwd_launch(const void* q, const void* k, const void* v, const void* o, const float* lse,
               const void* dout, void* dq, void* dk, void* dv, const fa::bwd::BParams& bp,
               float* dqacc, float* lse2, float* dsum, cudaStream_t st, DeviceInfo& info, int slot) {
  using L = fa::bwd::BLayout<D>;
  auto kern = fa::bwd::fa_bwd_kernel<D, BF16>;
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!info.bwd_attr_set[slot]) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES) !=
          cudaSuccess)
        return fail(FA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(cudaGetLastError()));
      cudaFuncAttributes fa_attr;
      if (cudaFuncGetAttributes(&fa_attr, kern) != cudaSuccess)
        return fail(FA_ERR_CUDA, "cudaFuncGetAttributes: %s", cudaGetErrorString(cudaGetLastError()));
      // The setmaxnreg split (2×136 + 144 + 96 per 128 threads) needs exactly
      // 128 registers per thread at launch.
      if (fa_attr.numRegs != 128)
        return fail(FA_ERR_UNSUPPORTED, "backward kernel built with %d registers per thread, need 128",
                    fa_attr.numRegs);
      info.bwd_attr_set[slot] = true;
    }
  }
  const long long BH = (long long)bp.B * bp.Hq;
  CUtensorMap tq, tk, tv, tdo;
  int rc;
  if ((rc = make_map(&tq, q, BF16, D, bp.N, BH, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK) return rc;
  if ((rc = make_map(&tk, k, BF16, D, bp.N, (long long)bp.B * bp.Hk, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK) return rc;
  if ((rc = make_map(&tv, v, BF16, D, bp.N, (long long)bp.B * bp.Hk, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK) return rc;
  if ((rc = make_map(&tdo, dout, BF16, D, bp.N, BH, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK)
    return rc;
  // fp32 dQ accumulator [B·Hq][N][D], reduced into in 32-column × 32-row boxes
  CUtensorMap tdq;
  {
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)bp.N, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)D * 4 * (cuuint64_t)bp.N};
    const cuuint32_t box[3] = {32, 32, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = driver_fns().encode(&tdq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, dqacc, dims, strides,
                                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled (dQ) failed (%d)", (int)r);
  }
  const long long pre_rows = BH * bp.Npad;
  long long pre_blocks = (pre_rows + 7) / 8;
  if (pre_blocks > (long long)info.sms * 32) pre_blocks = (long long)info.sms * 32;
  fa::bwd::fa_bwd_pre_kernel<D, BF16><<<(unsigned)pre_blocks, 256, 0, st>>>(
      o, dout, lse, lse2, dsum, dqacc, BH, bp.N, bp.Npad);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "backward prologue launch: %s", cudaGetErrorString(e));
  const int grid = bp.num_units < info.sms ? bp.num_units : info.sms;
  kern<<<grid, fa::bwd::NUM_THREADS, L::BYTES, st>>>(tq, tk, tv, tdo, tdq, bp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "backward launch: %s", cudaGetErrorString(e));
  const long long n8 = BH * bp.N * D / 8;
  long long post_blocks = (n8 + 255) / 256;
  if (post_blocks > (long long)info.sms * 32) post_blocks = (long long)info.sms * 32;
  fa::bwd::fa_bwd_post_kernel<BF16><<<(unsigned)post_blocks, 256, 0, st>>>(dqacc, dq, bp.scale, n8);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "backward epilogue launch: %s", cudaGetErrorString(e));
  return FA_OK;
}
}  // namespace

extern "C" size_t fa_bwd_workspace_bytes(int B, int Hq, int N, int d) {
  if (B < 1 || Hq < 1 || N < 1 || (d != 64 && d != 128)) return 0;
  return bwd_ws((long long)B * Hq, N, d).bytes;
}

extern "C" int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                      const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hk, int N,
                      int d, float scale, int causal, const int32_t* key_pad_lens, void* workspace,
                      size_t workspace_bytes, void* stream, int dtype) {
  g_err[0] = '\0';
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || lse == nullptr ||
      dout == nullptr || dq == nullptr || dk == nullptr || dv == nullptr)
    return fail(FA_ERR_INVALID_ARG, "q, k, v, o, lse, dout, dq, dk and dv must be non-NULL");
  if (B < 1 || Hq < 1 || Hk < 1 || N < 1)
    return fail(FA_ERR_INVALID_ARG, "B, Hq, Hk and N must be >= 1");
  if (Hq % Hk != 0) return fail(FA_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hk (%d)", Hq, Hk);
  if (d != 64 && d != 128)
    return fail(FA_ERR_UNSUPPORTED, "head dim %d not supported (64 or 128)", d);
  if (dtype != FA_FP16 && dtype != FA_BF16) return fail(FA_ERR_UNSUPPORTED, "unknown dtype %d", dtype);
  if (!std::isfinite(scale)) return fail(FA_ERR_INVALID_ARG, "scale must be finite");
  if (causal != 0 && causal != 1) return fail(FA_ERR_INVALID_ARG, "causal must be 0 or 1");
  const long long heads_q = (long long)B * Hq, heads_k = (long long)B * Hk;
  if (heads_q > 0x7fffffffLL || N > (1 << 30))
    return fail(FA_ERR_INVALID_ARG, "problem too large for 32-bit tile coordinates");
  const long long units = heads_k * ((N + 127) / 128);
  if (units > 0x7fffffffLL) return fail(FA_ERR_INVALID_ARG, "too many work units");
  const BwdWs ws = bwd_ws(heads_q, N, d);
  if (workspace_bytes < ws.bytes)
    return fail(FA_ERR_INVALID_ARG, "workspace of %zu bytes, need %zu", workspace_bytes, ws.bytes);
  // ---- device and buffers
  if (!driver_fns().ok) return fail(FA_ERR_CUDA, "CUDA driver entry points unavailable");
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return fail(FA_ERR_CUDA, "no current CUDA device");
  DeviceInfo& info = g_dev[dev];
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!info.init) {
      cudaDeviceProp prop;
      if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess)
        return fail(FA_ERR_CUDA, "cudaGetDeviceProperties failed");
      info.sm100 = prop.major == 10 && prop.minor == 0;
      info.sms = prop.multiProcessorCount;
      info.l2_bytes = prop.l2CacheSize;
      info.init = true;
    }
  }
  if (!info.sm100) return fail(FA_ERR_UNSUPPORTED, "device %d is not sm_100", dev);
  const size_t q_bytes = (size_t)heads_q * N * d * 2, kv_bytes = (size_t)heads_k * N * d * 2;
  const size_t lse_bytes = (size_t)heads_q * N * 4;
  int rc;
  if ((rc = check_range("q", q, q_bytes, 16)) != FA_OK) return rc;
  if ((rc = check_range("k", k, kv_bytes, 16)) != FA_OK) return rc;
  if ((rc = check_range("v", v, kv_bytes, 16)) != FA_OK) return rc;
  if ((rc = check_range("o", o, q_bytes, 16)) != FA_OK) return rc;
  if ((rc = check_range("lse", lse, lse_bytes, 4)) != FA_OK) return rc;
  if ((rc = check_range("dout", dout, q_bytes, 16)) != FA_OK) return rc;
  if ((rc = check_range("dq", dq, q_bytes, 16)) != FA_OK) return rc;
  if ((rc = check_range("dk", dk, kv_bytes, 16)) != FA_OK) return rc;
  if ((rc = check_range("dv", dv, kv_bytes, 16)) != FA_OK) return rc;
  if ((rc = check_range("workspace", workspace, ws.bytes, 256)) != FA_OK) return rc;
  if (key_pad_lens != nullptr &&
      (rc = check_range("key_pad_lens", key_pad_lens, (size_t)B * 4, 4)) != FA_OK)
    return rc;
  // outputs and the workspace may overlap nothing else
  struct Span { const void* p; size_t n; };
  const Span outs[4] = {{dq, q_bytes}, {dk, kv_bytes}, {dv, kv_bytes}, {workspace, ws.bytes}};
  const Span all[10] = {{q, q_bytes}, {k, kv_bytes}, {v, kv_bytes}, {o, q_bytes}, {lse, lse_bytes},
                        {dout, q_bytes}, {dq, q_bytes}, {dk, kv_bytes}, {dv, kv_bytes},
                        {workspace, ws.bytes}};
  for (int i = 0; i < 4; ++i)
    for (int j = 0; j < 10; ++j) {
      if (outs[i].p == all[j].p && outs[i].n == all[j].n && (j == 6 + i)) continue;  // itself
      const uintptr_t a = reinterpret_cast<uintptr_t>(outs[i].p), b = reinterpret_cast<uintptr_t>(all[j].p);
      if (a < b + all[j].n && b < a + outs[i].n)
        return fail(FA_ERR_INVALID_ARG, "an output or the workspace overlaps another argument");
    }
  fa::bwd::BParams bp;
  bp.B = B; bp.Hq = Hq; bp.Hk = Hk; bp.N = N; bp.G = Hq / Hk;
  bp.NM = (N + 127) / 128;
  bp.Npad = bp.NM * 128;
  bp.causal = causal;
  bp.num_units = (int)units;
  {
    // Head groups of the unit order: about 12 CTAs on each (b, hk) head at a
    // time, so that they share its Q and dO tiles in L2. Only causal problems
    // of at least eight waves of units, each group at least four waves, and
    // only when fewer than 12 CTAs per head are in flight without groups
    // (more CTAs on one head's tiles contend for the same L2 lines).
    bp.ng = 0;
    const long long grid = bp.num_units < info.sms ? bp.num_units : info.sms;
    const long long heads = heads_k, nkb = (N + 127) / 128;
    const long long per_group = grid / 12 > 0 ? grid / 12 : 1;
    if (causal && heads * nkb >= 8 * grid && heads > per_group) {
      long long ng = (heads + per_group - 1) / per_group;
      const long long min_heads = (4 * grid + nkb - 1) / nkb;
      if (ng > heads / min_heads) ng = heads / min_heads;
      bp.ng = ng > 1 ? (int)ng : 0;
    }
  }
  bp.key_pad_lens = key_pad_lens;
  uint8_t* wsb = reinterpret_cast<uint8_t*>(workspace);
  float* dqacc = reinterpret_cast<float*>(wsb + ws.dq_off);
  float* lse2 = reinterpret_cast<float*>(wsb + ws.lse2_off);
  float* dsum = reinterpret_cast<float*>(wsb + ws.dsum_off);
  bp.lse2 = lse2;
  bp.dsum = dsum;
  bp.dqacc = dqacc;
  bp.dk = dk;
  bp.dv = dv;
  bp.scale_log2 = (float)((double)scale * 1.4426950408889634);
  bp.scale = scale;
  bp.timeout_ns = g_timeout_ns;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf16 = dtype == FA_BF16;
  if (d == 128)
    return bf16 ? bwd_launch<128, true>(q, k, v, o, lse, dout, dq, dk, dv, bp, dqacc, lse2, dsum, st, info, 0)
                : bwd_launch<128, false>(q, k, v, o, lse, dout, dq, dk, dv, bp, dqacc, lse2, dsum, st, info, 1);
  return bf16 ? bwd_launch<64, true>(q, k, v, o, lse, dout, dq, dk, dv, bp, dqacc, lse2, dsum, st, info, 2)
              : bwd_launch<64, false>(q, k, v, o, lse, dout, dq, dk, dv, bp, dqacc, lse2, dsum, st, info, 3);
}

// ============================================================= FP8 forward
namespace {
size_t fp8_ws_bytes(long long heads_k, int N, int d) {
  return ((size_t)heads_k * N * d + 255) / 256 * 256;
}
}  // namespace

extern "C" size_t fa_fwd_fp8_workspace_bytes(int B, int Hk, int N, int d) {
  if (B < 1 || Hk < 1 || N < 1 || d != 128) return 0;
  return fp8_ws_bytes((long long)B * Hk, N, d);
}

extern "C" int fa_fwd_fp8(const void* q, const void* k, const void* v, float q_descale,
                          float k_descale, float v_descale, void* o, float* lse, int B, int Hq,
                          int Hk, int N, int d, float scale, int causal,
                          const int32_t* key_pad_lens, void* workspace, size_t workspace_bytes,
                          void* stream) {
  g_err[0] = '\0';
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr)
    return fail(FA_ERR_INVALID_ARG, "q, k, v and o must be non-NULL");
  if (B < 1 || Hq < 1 || Hk < 1 || N < 1)
    return fail(FA_ERR_INVALID_ARG, "B, Hq, Hk and N must be >= 1");
  if (Hq % Hk != 0) return fail(FA_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hk (%d)", Hq, Hk);
  if (d != 128) return fail(FA_ERR_UNSUPPORTED, "FP8 forward supports head dim 128, not %d", d);
  if (N % 16 != 0)
    return fail(FA_ERR_UNSUPPORTED, "FP8 forward needs N %% 16 == 0 (16-byte rows of Vᵀ), N = %d", N);
  if (!std::isfinite(scale)) return fail(FA_ERR_INVALID_ARG, "scale must be finite");
  if (!(std::isfinite(q_descale) && std::isfinite(k_descale) && std::isfinite(v_descale)) ||
      q_descale <= 0.f || k_descale <= 0.f || v_descale <= 0.f)
    return fail(FA_ERR_INVALID_ARG, "descale factors must be finite and > 0");
  if (causal != 0 && causal != 1) return fail(FA_ERR_INVALID_ARG, "causal must be 0 or 1");
  const long long heads_q = (long long)B * Hq, heads_k = (long long)B * Hk;
  if (heads_q > 0x7fffffffLL || N > (1 << 30))
    return fail(FA_ERR_INVALID_ARG, "problem too large for 32-bit tile coordinates");
  if (fa_num_units(B, Hq, Hk, N, causal) < 0) return FA_ERR_INVALID_ARG;
  const size_t need = fp8_ws_bytes(heads_k, N, d);
  if (workspace_bytes < need)
    return fail(FA_ERR_INVALID_ARG, "workspace of %zu bytes, need %zu", workspace_bytes, need);
  if (!driver_fns().ok) return fail(FA_ERR_CUDA, "CUDA driver entry points unavailable");
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return fail(FA_ERR_CUDA, "no current CUDA device");
  DeviceInfo& info = g_dev[dev];
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!info.init) {
      cudaDeviceProp prop;
      if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess)
        return fail(FA_ERR_CUDA, "cudaGetDeviceProperties failed");
      info.sm100 = prop.major == 10 && prop.minor == 0;
      info.sms = prop.multiProcessorCount;
      info.l2_bytes = prop.l2CacheSize;
      info.init = true;
    }
  }
  if (!info.sm100) return fail(FA_ERR_UNSUPPORTED, "device %d is not sm_100", dev);
  const size_t q_bytes = (size_t)heads_q * N * d, kv_bytes = (size_t)heads_k * N * d;
  const size_t o_bytes = q_bytes * 2, lse_bytes = (size_t)heads_q * N * 4;
  int rc;
  if ((rc = check_range("q", q, q_bytes, 16)) != FA_OK) return rc;
  if ((rc = check_range("k", k, kv_bytes, 16)) != FA_OK) return rc;
  if ((rc = check_range("v", v, kv_bytes, 16)) != FA_OK) return rc;
  if ((rc = check_range("o", o, o_bytes, 16)) != FA_OK) return rc;
  if (lse != nullptr && (rc = check_range("lse", lse, lse_bytes, 4)) != FA_OK) return rc;
  if ((rc = check_range("workspace", workspace, need, 256)) != FA_OK) return rc;
  if (key_pad_lens != nullptr &&
      (rc = check_range("key_pad_lens", key_pad_lens, (size_t)B * 4, 4)) != FA_OK)
    return rc;
  struct Span { const void* p; size_t n; };
  const Span outs[3] = {{o, o_bytes}, {lse, lse_bytes}, {workspace, need}};
  const Span all[6] = {{q, q_bytes}, {k, kv_bytes}, {v, kv_bytes}, {o, o_bytes}, {lse, lse_bytes},
                       {workspace, need}};
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 6; ++j) {
      if (j == 3 + i || outs[i].p == nullptr || all[j].p == nullptr) continue;
      const uintptr_t a = reinterpret_cast<uintptr_t>(outs[i].p), b = reinterpret_cast<uintptr_t>(all[j].p);
      if (a < b + all[j].n && b < a + outs[i].n)
        return fail(FA_ERR_INVALID_ARG, "an output or the workspace overlaps another argument");
    }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* vt = reinterpret_cast<uint8_t*>(workspace);
  const dim3 tgrid((unsigned)((N + 63) / 64), (unsigned)(d / 64), (unsigned)heads_k);
  fa::fa_transpose_u8_kernel<<<tgrid, 256, 0, st>>>(reinterpret_cast<const uint8_t*>(v), vt, N, d);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "V transpose launch: %s", cudaGetErrorString(e));
  fa::Params prm;
  prm.key_pad_lens = key_pad_lens;
  prm.lse = lse;
  prm.o_part = nullptr;
  prm.lse_part = nullptr;
  prm.o_scale = v_descale;
  prm.bias_bmul = 0;
  prm.bias_hmul = 0;
  prm.bias_H = 1;
  prm.s = fa::make_shape(B, Hq, Hk, N, causal, 1);
  prm.scale_log2 = (float)((double)scale * q_descale * k_descale * 1.4426950408889634);
  prm.timeout_ns = g_timeout_ns;
  return launch<128, true, 2>(q, k, vt, o, prm, st, info, 8, lse);
}

#include "fa_host_pipeline.cuh"
