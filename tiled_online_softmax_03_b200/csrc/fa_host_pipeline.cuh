// fa_host_pipeline.cuh — fa_fwd_host: the attention forward on host buffers.
//
// The user-level call of the pages takes whole Q, K, V tensors and returns O
// (the NPU page "FlashAttention 在昇腾 NPU 上是怎么省显存的？我花了两天把它搞明白
// 了", usage section: flash_attention(q, k, v, block_size, causal)). With the
// tensors in host memory the PCIe copies cost more than the attention itself,
// so the work is cut into chunks of whole (b, K/V head) groups and, per chunk,
// the copy in, the attention and the copy out run on three streams: the two
// PCIe directions and the kernel overlap. Included once, at the end of
// fa_fwd_sm100.cu (it uses that file's validation and launch path).

namespace {

constexpr int FA_HOST_MAX_CHUNKS = 64;
constexpr double FA_HOST_CHUNK_BYTES = 16.0 * (1 << 20);  // target copy-in bytes per chunk

struct HostChunk {
  int b0, b1;    // batches [b0, b1)
  int hk0, hk1;  // K/V heads [hk0, hk1) of each of those batches (all heads when b1 - b0 > 1)
};

// Chunk plan: `want` chunks (0: about 16 MB of inputs per chunk, at most 16),
// as near-equal runs of whole batches when B >= want, else every batch cut
// into near-equal runs of K/V heads (each with its query heads), so that one
// chunk is always one contiguous slice of q, k, v, o and lse.
int host_chunk_plan(int B, int Hq, int Hk, int N, int d, int want, HostChunk* out, int max_out) {
  if (want <= 0) {
    const double in_bytes = 2.0 * B * (double)N * d * (Hq + 2.0 * Hk);
    want = (int)(in_bytes / FA_HOST_CHUNK_BYTES);
    want = want < 1 ? 1 : (want > 16 ? 16 : want);
  }
  if (want > max_out) want = max_out;
  int n = 0;
  if (B >= want) {
    const int base = B / want, extra = B % want;
    int b0 = 0;
    for (int i = 0; i < want; ++i) {
      const int b1 = b0 + base + (i < extra ? 1 : 0);
      out[n++] = HostChunk{b0, b1, 0, Hk};
      b0 = b1;
    }
    return n;
  }
  int per_b = (want + B - 1) / B;
  if (per_b > Hk) per_b = Hk;
  if (per_b * B > max_out) per_b = max_out / B;
  if (per_b < 1) per_b = 1;
  const int base = Hk / per_b, extra = Hk % per_b;
  for (int b = 0; b < B; ++b) {
    int h0 = 0;
    for (int i = 0; i < per_b; ++i) {
      const int h1 = h0 + base + (i < extra ? 1 : 0);
      out[n++] = HostChunk{b, b + 1, h0, h1};
      h0 = h1;
    }
  }
  return n;
}

// Two copy streams per device (copies in, copies out), created on first use
// and kept for the life of the process; created again if the current context
// changed (a new primary context after cudaDeviceReset).
struct CopyStreams {
  CUcontext ctx = nullptr;
  cudaStream_t in = nullptr, out = nullptr;
};
CopyStreams g_copy_streams[64];

int copy_streams(int dev, cudaStream_t* s_in, cudaStream_t* s_out) {
  CUcontext ctx = nullptr;
  if (driver_fns().ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
    return fail(FA_ERR_CUDA, "no current CUDA context");
  std::lock_guard<std::mutex> lk(g_dev_mu);
  CopyStreams& c = g_copy_streams[dev];
  if (c.in == nullptr || c.ctx != ctx) {
    cudaStream_t a = nullptr, b = nullptr;
    if (cudaStreamCreateWithFlags(&a, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&b, cudaStreamNonBlocking) != cudaSuccess)
      return fail(FA_ERR_CUDA, "creating the copy streams: %s",
                  cudaGetErrorString(cudaGetLastError()));
    c.ctx = ctx;
    c.in = a;
    c.out = b;
  }
  *s_in = c.in;
  *s_out = c.out;
  return FA_OK;
}

// Host memory that copies can run from asynchronously: pinned (page-locked or
// registered) memory of the current context.
int check_pinned(const char* name, const void* ptr) {
  if (ptr == nullptr) return fail(FA_ERR_INVALID_ARG, "%s is NULL", name);
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
    cudaGetLastError();
    return fail(FA_ERR_INVALID_ARG, "%s: not a pointer CUDA knows", name);
  }
  if (a.type != cudaMemoryTypeHost)
    return fail(FA_ERR_INVALID_ARG, "%s must be pinned host memory (cudaMallocHost or registered)",
                name);
  return FA_OK;
}

}  // namespace

extern "C" int fa_host_chunk_plan(int B, int Hq, int Hk, int N, int d, int num_chunks, int32_t* out,
                                  int max_chunks) {
  if (B < 1 || Hq < 1 || Hk < 1 || N < 1 || d < 1 || Hq % Hk != 0)
    return fail(FA_ERR_INVALID_ARG, "bad shape");
  if (num_chunks < 0 || num_chunks > FA_HOST_MAX_CHUNKS)
    return fail(FA_ERR_INVALID_ARG, "num_chunks %d out of [0, %d]", num_chunks, FA_HOST_MAX_CHUNKS);
  if (out == nullptr || max_chunks < 1) return fail(FA_ERR_INVALID_ARG, "no room for the plan");
  HostChunk plan[FA_HOST_MAX_CHUNKS];
  const int n = host_chunk_plan(B, Hq, Hk, N, d, num_chunks, plan,
                                max_chunks < FA_HOST_MAX_CHUNKS ? max_chunks : FA_HOST_MAX_CHUNKS);
  for (int i = 0; i < n; ++i) {
    out[4 * i] = plan[i].b0;
    out[4 * i + 1] = plan[i].b1;
    out[4 * i + 2] = plan[i].hk0;
    out[4 * i + 3] = plan[i].hk1;
  }
  return n;
}

extern "C" int fa_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                           int Hq, int Hk, int N, int d, float scale, int causal,
                           const int32_t* key_pad_lens, void* q_dev, void* k_dev, void* v_dev,
                           void* o_dev, float* lse_dev, int32_t* lens_dev, int num_chunks,
                           void* stream, int dtype) {
  g_err[0] = '\0';
  // ---- arguments that need no CUDA call
  if (B < 1 || Hq < 1 || Hk < 1 || N < 1)
    return fail(FA_ERR_INVALID_ARG, "B, Hq, Hk and N must be >= 1");
  if (Hq % Hk != 0) return fail(FA_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hk (%d)", Hq, Hk);
  if (d != 64 && d != 128)
    return fail(FA_ERR_UNSUPPORTED, "head dim %d not supported (64 or 128)", d);
  if (dtype != FA_FP16 && dtype != FA_BF16) return fail(FA_ERR_UNSUPPORTED, "unknown dtype %d", dtype);
  if (num_chunks < 0 || num_chunks > FA_HOST_MAX_CHUNKS)
    return fail(FA_ERR_INVALID_ARG, "num_chunks %d out of [0, %d]", num_chunks, FA_HOST_MAX_CHUNKS);
  if ((lse == nullptr) != (lse_dev == nullptr))
    return fail(FA_ERR_INVALID_ARG, "lse and lse_dev must both be given or both be NULL");
  if (key_pad_lens != nullptr && lens_dev == nullptr)
    return fail(FA_ERR_INVALID_ARG, "key_pad_lens needs a device buffer lens_dev");
  const long long heads_q = (long long)B * Hq, heads_k = (long long)B * Hk;
  if (heads_q > 0x7fffffffLL || N > (1 << 30))
    return fail(FA_ERR_INVALID_ARG, "problem too large for 32-bit tile coordinates");
  // ---- host and device buffers
  if (!driver_fns().ok) return fail(FA_ERR_CUDA, "CUDA driver entry points unavailable");
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return fail(FA_ERR_CUDA, "no current CUDA device");
  int rc;
  if ((rc = check_pinned("q", q)) != FA_OK || (rc = check_pinned("k", k)) != FA_OK ||
      (rc = check_pinned("v", v)) != FA_OK || (rc = check_pinned("o", o)) != FA_OK)
    return rc;
  if (lse != nullptr && (rc = check_pinned("lse", lse)) != FA_OK) return rc;
  if (key_pad_lens != nullptr && (rc = check_pinned("key_pad_lens", key_pad_lens)) != FA_OK) return rc;
  const size_t el = 2, q_bytes = (size_t)heads_q * N * d * el, kv_bytes = (size_t)heads_k * N * d * el;
  const size_t lse_bytes = (size_t)heads_q * N * 4;
  if ((rc = check_range("q_dev", q_dev, q_bytes, 16)) != FA_OK) return rc;
  if ((rc = check_range("k_dev", k_dev, kv_bytes, 16)) != FA_OK) return rc;
  if ((rc = check_range("v_dev", v_dev, kv_bytes, 16)) != FA_OK) return rc;
  if ((rc = check_range("o_dev", o_dev, q_bytes, 16)) != FA_OK) return rc;
  if (lse_dev != nullptr && (rc = check_range("lse_dev", lse_dev, lse_bytes, 4)) != FA_OK) return rc;
  if (key_pad_lens != nullptr && (rc = check_range("lens_dev", lens_dev, (size_t)B * 4, 4)) != FA_OK)
    return rc;
  {
    // the device buffers are written by the copies in: none may overlap another
    struct Span { const void* p; size_t n; };
    const Span sp[6] = {{q_dev, q_bytes}, {k_dev, kv_bytes}, {v_dev, kv_bytes}, {o_dev, q_bytes},
                        {lse_dev, lse_bytes}, {key_pad_lens ? lens_dev : nullptr, (size_t)B * 4}};
    for (int i = 0; i < 6; ++i)
      for (int j = i + 1; j < 6; ++j) {
        if (sp[i].p == nullptr || sp[j].p == nullptr) continue;
        const uintptr_t a = reinterpret_cast<uintptr_t>(sp[i].p), b = reinterpret_cast<uintptr_t>(sp[j].p);
        if (a < b + sp[j].n && b < a + sp[i].n)
          return fail(FA_ERR_INVALID_ARG, "device buffers overlap");
      }
  }
  cudaStream_t s_in = nullptr, s_out = nullptr;
  if ((rc = copy_streams(dev, &s_in, &s_out)) != FA_OK) return rc;
  HostChunk plan[FA_HOST_MAX_CHUNKS];
  const int nch = host_chunk_plan(B, Hq, Hk, N, d, num_chunks, plan, FA_HOST_MAX_CHUNKS);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  cudaEvent_t ev_fork = nullptr, ev_in = nullptr, ev_k = nullptr, ev_join = nullptr;
  if (cudaEventCreateWithFlags(&ev_fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&ev_in, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&ev_k, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&ev_join, cudaEventDisableTiming) != cudaSuccess) {
    cudaGetLastError();
    for (cudaEvent_t e : {ev_fork, ev_in, ev_k, ev_join})
      if (e != nullptr) cudaEventDestroy(e);
    return fail(FA_ERR_CUDA, "creating events failed");
  }
  const int G = Hq / Hk;
  const size_t head_elems = (size_t)N * d;
  auto cuda_ok = [&](cudaError_t e, const char* what) {
    if (e == cudaSuccess) return true;
    rc = fail(FA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return false;
  };
  // Everything earlier on the caller's stream (a previous call's copies out
  // included, which that stream waits for) comes first: the device buffers
  // are reused.
  rc = FA_OK;
  bool ok = cuda_ok(cudaEventRecord(ev_fork, cs), "event record") &&
            cuda_ok(cudaStreamWaitEvent(s_in, ev_fork, 0), "stream wait") &&
            cuda_ok(cudaStreamWaitEvent(s_out, ev_fork, 0), "stream wait");
  if (ok && key_pad_lens != nullptr)
    ok = cuda_ok(cudaMemcpyAsync(lens_dev, key_pad_lens, (size_t)B * 4, cudaMemcpyHostToDevice, s_in),
                 "copy in");
  const uint8_t* qh = static_cast<const uint8_t*>(q);
  const uint8_t* kh = static_cast<const uint8_t*>(k);
  const uint8_t* vh = static_cast<const uint8_t*>(v);
  uint8_t* oh = static_cast<uint8_t*>(o);
  uint8_t* qd = static_cast<uint8_t*>(q_dev);
  uint8_t* kd = static_cast<uint8_t*>(k_dev);
  uint8_t* vd = static_cast<uint8_t*>(v_dev);
  uint8_t* od = static_cast<uint8_t*>(o_dev);
  for (int c = 0; ok && c < nch; ++c) {
    const HostChunk& ch = plan[c];
    const int cb = ch.b1 - ch.b0, chk = ch.hk1 - ch.hk0;
    // first query / K/V head of the chunk, as a flat head index
    const size_t hq0 = (size_t)ch.b0 * Hq + (size_t)ch.hk0 * G;
    const size_t hk0 = (size_t)ch.b0 * Hk + ch.hk0;
    const size_t nq = (size_t)cb * chk * G, nk = (size_t)cb * chk;
    const size_t qoff = hq0 * head_elems * el, qlen = nq * head_elems * el;
    const size_t koff = hk0 * head_elems * el, klen = nk * head_elems * el;
    ok = cuda_ok(cudaMemcpyAsync(qd + qoff, qh + qoff, qlen, cudaMemcpyHostToDevice, s_in), "copy in") &&
         cuda_ok(cudaMemcpyAsync(kd + koff, kh + koff, klen, cudaMemcpyHostToDevice, s_in), "copy in") &&
         cuda_ok(cudaMemcpyAsync(vd + koff, vh + koff, klen, cudaMemcpyHostToDevice, s_in), "copy in") &&
         cuda_ok(cudaEventRecord(ev_in, s_in), "event record") &&
         cuda_ok(cudaStreamWaitEvent(cs, ev_in, 0), "stream wait");
    if (!ok) break;
    float* lse_c = lse_dev != nullptr ? lse_dev + hq0 * N : nullptr;
    rc = fwd_impl(qd + qoff, kd + koff, vd + koff, od + qoff, lse_c, cb, chk * G, chk, N, d, scale,
                  causal, key_pad_lens != nullptr ? lens_dev + ch.b0 : nullptr, 1, nullptr, 0, cs,
                  dtype);
    if (rc != FA_OK) {
      ok = false;
      break;
    }
    ok = cuda_ok(cudaEventRecord(ev_k, cs), "event record") &&
         cuda_ok(cudaStreamWaitEvent(s_out, ev_k, 0), "stream wait") &&
         cuda_ok(cudaMemcpyAsync(oh + qoff, od + qoff, qlen, cudaMemcpyDeviceToHost, s_out), "copy out");
    if (ok && lse != nullptr)
      ok = cuda_ok(cudaMemcpyAsync(lse + hq0 * N, lse_c, nq * N * 4, cudaMemcpyDeviceToHost, s_out),
                   "copy out");
  }
  // Join: the caller's stream waits for every copy, also after an error, so
  // that nothing enqueued here outlives what the caller synchronises on.
  const int rc_loop = rc;
  const cudaError_t j1 = cudaEventRecord(ev_join, s_in);
  const cudaError_t j2 = j1 == cudaSuccess ? cudaStreamWaitEvent(cs, ev_join, 0) : j1;
  const cudaError_t j3 = cudaEventRecord(ev_join, s_out);
  const cudaError_t j4 = j3 == cudaSuccess ? cudaStreamWaitEvent(cs, ev_join, 0) : j3;
  for (cudaEvent_t e : {ev_fork, ev_in, ev_k, ev_join}) cudaEventDestroy(e);
  if (rc_loop != FA_OK) return rc_loop;
  if (j2 != cudaSuccess || j4 != cudaSuccess)
    return fail(FA_ERR_CUDA, "joining the copy streams: %s",
                cudaGetErrorString(j2 != cudaSuccess ? j2 : j4));
  return FA_OK;
}
