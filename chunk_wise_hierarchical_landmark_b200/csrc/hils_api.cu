// C ABI of libhils.so (declared in include/hils.h): argument validation,
// workspace sizing, kernel dispatch and status reporting.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "../../include/hils.h"
#include "kernels.h"
#include "hope.h"
#include "paged.h"
#include "qcal.h"
#include "backward.h"

#define HILS_API extern "C" __attribute__((visibility("default")))

namespace {

std::atomic<int64_t> g_launches{0};
thread_local char g_msg[256] = "";

hils_status fail(hils_status s, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
hils_status fail(hils_status s, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof g_msg, fmt, ap);
  va_end(ap);
  return s;
}

hils_status cuda_fail(cudaError_t e, const char *where) {
  return fail(HILS_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

constexpr int kMaxL = 1 << 24;
constexpr size_t kDebugWs = 256;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

hils_status check_params(const hils_params *p) {
  if (!p) return fail(HILS_ERR_INVALID_ARG, "params is NULL");
  if (p->B < 1 || p->Hq < 1 || p->Hkv < 1 || p->L < 1 || p->d < 1 || p->chunk < 1 ||
      p->topk < 1 || p->M < 1)
    return fail(HILS_ERR_INVALID_ARG, "shape fields must be >= 1");
  if (p->Hq % p->Hkv) return fail(HILS_ERR_INVALID_ARG, "Hq %% Hkv != 0");
  if (!std::isfinite(p->scale) || !(p->scale > 0.0f))
    return fail(HILS_ERR_INVALID_ARG, "scale must be finite and positive");
  if (p->dtype != HILS_F32 && p->dtype != HILS_BF16)
    return fail(HILS_ERR_INVALID_ARG, "unknown dtype %d", p->dtype);
  if (p->debug_checks != 0 && p->debug_checks != 1)
    return fail(HILS_ERR_INVALID_ARG, "debug_checks must be 0 or 1");
  if (p->d != 64 && p->d != 128) return fail(HILS_ERR_UNSUPPORTED, "d=%d (supported: 64, 128)", p->d);
  if (p->chunk != 64) return fail(HILS_ERR_UNSUPPORTED, "chunk=%d (supported: 64)", p->chunk);
  if (p->topk > 64) return fail(HILS_ERR_UNSUPPORTED, "topk=%d (supported: 1..64)", p->topk);
  if (p->M != 16 && p->M != 32 && p->M != 64 && p->M != 128)
    return fail(HILS_ERR_UNSUPPORTED, "M=%d (supported: 16, 32, 64, 128)", p->M);
  if (p->L > kMaxL) return fail(HILS_ERR_UNSUPPORTED, "L=%d above %d", p->L, kMaxL);
  if ((int64_t)p->B * p->Hq > (1 << 16) - 1)
    return fail(HILS_ERR_UNSUPPORTED, "B*Hq above 65535");
  if ((int64_t)p->B * p->Hq * p->L >= (int64_t)1 << 31)
    return fail(HILS_ERR_UNSUPPORTED, "B*Hq*L must be below 2^31");
  return HILS_OK;
}

#define NEED(ptr)                                                              \
  do {                                                                         \
    if (!(ptr)) return fail(HILS_ERR_INVALID_ARG, #ptr " is NULL");            \
    if (!aligned16(ptr)) return fail(HILS_ERR_INVALID_ARG, #ptr " is not 16-byte aligned"); \
  } while (0)
#define MAYBE(ptr)                                                             \
  do {                                                                         \
    if ((ptr) && !aligned16(ptr)) return fail(HILS_ERR_INVALID_ARG, #ptr " is not 16-byte aligned"); \
  } while (0)

// Failure-path test settings (hils_test_set_wait_limit); 0 = the default limit.
std::atomic<unsigned long long> g_test_wait_ns{0};
std::atomic<int> g_test_withhold{0};

hils::RowSpec prefill_rows(const hils_params *p) {
  hils::RowSpec rs{p->B, p->Hq, p->Hkv, p->L, p->d, p->chunk, p->topk, p->scale, 0, p->L};
  const unsigned long long ns = g_test_wait_ns.load();
  if (ns) rs.wait_ns = ns;
  rs.withhold = g_test_withhold.load();
  return rs;
}

// Debug mode: clear the device error word before the launches ...
hils_status debug_begin(const hils_params *p, void *ws, size_t ws_bytes, uint32_t **err,
                        cudaStream_t st) {
  *err = nullptr;
  if (!p->debug_checks) return HILS_OK;
  if (!ws || ws_bytes < kDebugWs) return fail(HILS_ERR_WORKSPACE, "debug_checks needs %zu bytes of workspace", kDebugWs);
  *err = static_cast<uint32_t *>(ws);
  cudaError_t e = cudaMemsetAsync(*err, 0, sizeof(uint32_t), st);
  return e == cudaSuccess ? HILS_OK : cuda_fail(e, "cudaMemsetAsync");
}
// ... and read it back (synchronising the stream) after them.
hils_status debug_end(uint32_t *err, cudaStream_t st) {
  if (!err) return HILS_OK;
  uint32_t code = 0;
  cudaError_t e = cudaMemcpyAsync(&code, err, sizeof code, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "debug read-back");
  if (code == 5) return fail(HILS_ERR_DEVICE_CHECK, "a device-side check found an invalid chunk index");
  if (code == 6) return fail(HILS_ERR_TIMEOUT, "a bounded device wait gave up");
  if (code) return fail(HILS_ERR_DEVICE_CHECK, "device error word %u", code);
  return HILS_OK;
}

const hils::HopeParams kNoHope{};

hils_status do_select(const hils_params *p, const hils::RowSpec &rs, const void *q,
                      const void *lmk, int32_t *sel, float *w, float *lse_lmk, uint32_t *err,
                      cudaStream_t st, const hils::HopeParams &hp = kNoHope) {
  // bf16 prefill scores on the tensor cores; fp32 and the decode row on the CUDA cores
  const bool tc = p->dtype == HILS_BF16 && rs.t_first == 0 && rs.t_count == rs.L;
  int n = 0;
  cudaError_t e;
  if (tc) {
    e = hils::select_sm100(rs, q, lmk, sel, w, lse_lmk, err, st, &n, hp);
  } else {
    e = hils::select_simt(rs, p->dtype == HILS_BF16, q, lmk, sel, w, lse_lmk, st);
    n = 1;
  }
  g_launches += n;
  return e == cudaSuccess ? HILS_OK : cuda_fail(e, "select launch");
}

hils_status do_attn(const hils_params *p, const hils::RowSpec &rs, const void *q, const void *k,
                    const void *v, const int32_t *sel, const float *w, void *out, float *lse,
                    float *wfin, uint32_t *err, cudaStream_t st,
                    const hils::HopeParams &hp = kNoHope) {
  // bf16 prefill runs on the tensor cores; fp32 (no exact tensor-core path)
  // and the single decode row run on the CUDA cores
  const bool tc = p->dtype == HILS_BF16 && rs.t_first == 0 && rs.t_count == rs.L;
  cudaError_t e = tc ? hils::attn_sm100(rs, q, k, v, sel, w, out, lse, wfin, err, st, hp)
                     : hils::attn_simt(rs, p->dtype == HILS_BF16, q, k, v, sel, w, out, lse,
                                       wfin, err, st);
  g_launches += 1;
  return e == cudaSuccess ? HILS_OK : cuda_fail(e, "attention launch");
}

hils::DecodeSpec decode_spec_of(const hils_params *p) {
  return hils::decode_spec(p->B, p->Hq, p->Hkv, p->L, p->d, p->topk, p->scale);
}

hils_status check_decode(const hils_params *p) {
  if ((size_t)(p->Hq / p->Hkv) > hils::decode_max_g())
    return fail(HILS_ERR_UNSUPPORTED, "decode supports Hq/Hkv <= %zu", hils::decode_max_g());
  return HILS_OK;
}

}  // namespace

HILS_API size_t hils_workspace_size(const hils_params *p, int op) {
  if (check_params(p) != HILS_OK) return 0;
  if (op == HILS_OP_PREFILL) return p->debug_checks ? kDebugWs : 0;
  if (op == HILS_OP_DECODE) {
    if (check_decode(p) != HILS_OK) return 0;
    return hils::decode_workspace_bytes(decode_spec_of(p));
  }
  return 0;
}

HILS_API hils_status hils_select(const hils_params *p, const void *q, const void *lmk_k,
                                 int32_t *sel_idx, float *chunk_w, float *lse_lmk, void *ws,
                                 size_t ws_bytes, void *stream) {
  hils_status s = check_params(p);
  if (s != HILS_OK) return s;
  NEED(q);
  NEED(sel_idx);
  NEED(chunk_w);
  MAYBE(lse_lmk);
  if (p->L >= p->chunk) NEED(lmk_k);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t *err = nullptr;
  if ((s = debug_begin(p, ws, ws_bytes, &err, st)) != HILS_OK) return s;
  if ((s = do_select(p, prefill_rows(p), q, lmk_k, sel_idx, chunk_w, lse_lmk, err, st)) != HILS_OK)
    return s;
  return debug_end(err, st);
}

HILS_API int64_t hils_union_capacity(const hils_params *p) {
  if (check_params(p) != HILS_OK) return -1;
  const int64_t nchunks = (p->L + p->chunk - 1) / p->chunk;
  const int64_t gph = (p->L + p->M - 1) / p->M;
  const int64_t per = std::min<int64_t>(nchunks, (int64_t)p->M * p->topk + p->M / p->chunk + 2);
  return (int64_t)p->B * p->Hq * gph * per;
}

HILS_API hils_status hils_union(const hils_params *p, const int32_t *sel_idx, int32_t *u_off,
                                int32_t *u_idx, int64_t u_cap, void *ws, size_t ws_bytes,
                                void *stream) {
  hils_status s = check_params(p);
  if (s != HILS_OK) return s;
  NEED(sel_idx);
  NEED(u_off);
  NEED(u_idx);
  if (u_cap < hils_union_capacity(p))
    return fail(HILS_ERR_INVALID_ARG, "u_cap %lld below hils_union_capacity", (long long)u_cap);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t *err = nullptr;
  if ((s = debug_begin(p, ws, ws_bytes, &err, st)) != HILS_OK) return s;
  int n = 0;
  cudaError_t e = hils::union_csr(p->B, p->Hq, p->L, p->chunk, p->topk, p->M, sel_idx, u_off,
                                  u_idx, u_cap, err, st, &n);
  g_launches += n;
  if (e != cudaSuccess) return cuda_fail(e, "union launch");
  return debug_end(err, st);
}

HILS_API hils_status hils_attn_fwd(const hils_params *p, const void *q, const void *k,
                                   const void *v, const int32_t *sel_idx, const float *chunk_w,
                                   void *out, float *lse, float *w_final, void *ws,
                                   size_t ws_bytes, void *stream) {
  hils_status s = check_params(p);
  if (s != HILS_OK) return s;
  NEED(q);
  NEED(k);
  NEED(v);
  NEED(sel_idx);
  NEED(chunk_w);
  NEED(out);
  NEED(lse);
  MAYBE(w_final);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t *err = nullptr;
  if ((s = debug_begin(p, ws, ws_bytes, &err, st)) != HILS_OK) return s;
  s = do_attn(p, prefill_rows(p), q, k, v, sel_idx, chunk_w, out, lse, w_final, err, st);
  if (s != HILS_OK) return s;
  return debug_end(err, st);
}

HILS_API hils_status hils_prefill(const hils_params *p, const void *q, const void *k,
                                  const void *v, const void *lmk_k, int32_t *sel_idx,
                                  float *chunk_w, float *lse_lmk, void *out, float *lse, void *ws,
                                  size_t ws_bytes, void *stream) {
  hils_status s = hils_select(p, q, lmk_k, sel_idx, chunk_w, lse_lmk, ws, ws_bytes, stream);
  if (s != HILS_OK) return s;
  return hils_attn_fwd(p, q, k, v, sel_idx, chunk_w, out, lse, nullptr, ws, ws_bytes, stream);
}

namespace {

// The decode step over dense caches (pages.table == nullptr) or paged ones.
hils_status decode_impl(const hils_params *p, const void *q, const void *k, const void *v,
                        const hils::PagedKV &pages, const void *lmk_k, int32_t *sel_idx,
                        float *chunk_w, float *lse_lmk, void *out, float *lse, void *ws,
                        size_t ws_bytes, void *stream) {
  hils_status s;
  NEED(sel_idx);
  NEED(chunk_w);
  NEED(out);
  NEED(lse);
  MAYBE(lse_lmk);
  if (p->L > p->chunk) NEED(lmk_k);
  if ((s = check_decode(p)) != HILS_OK) return s;
  const hils::DecodeSpec ds = decode_spec_of(p);
  const size_t need = hils::decode_workspace_bytes(ds);
  if (!ws || ws_bytes < need)
    return fail(HILS_ERR_WORKSPACE, "decode needs %zu bytes of workspace, got %zu", need, ws_bytes);
  NEED(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t *err = nullptr;
  if ((s = debug_begin(p, ws, ws_bytes, &err, st)) != HILS_OK) return s;
  int n = 0;
  cudaError_t e =
      pages.table ? hils::decode_fwd_paged(ds, p->dtype == HILS_BF16, q, k, v, pages, lmk_k,
                                           sel_idx, chunk_w, lse_lmk, out, lse, ws, err, st, &n)
                  : hils::decode_fwd(ds, p->dtype == HILS_BF16, q, k, v, lmk_k, sel_idx, chunk_w,
                                     lse_lmk, out, lse, ws, err, st, &n);
  g_launches += n;
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return debug_end(err, st);
}

}  // namespace

HILS_API hils_status hils_decode_fwd(const hils_params *p, const void *q, const void *k_cache,
                                     const void *v_cache, const void *lmk_k, int32_t *sel_idx,
                                     float *chunk_w, float *lse_lmk, void *out, float *lse,
                                     void *ws, size_t ws_bytes, void *stream) {
  hils_status s = check_params(p);
  if (s != HILS_OK) return s;
  NEED(q);
  NEED(k_cache);
  NEED(v_cache);
  return decode_impl(p, q, k_cache, v_cache, hils::PagedKV{nullptr, 0, 0}, lmk_k, sel_idx,
                     chunk_w, lse_lmk, out, lse, ws, ws_bytes, stream);
}

HILS_API hils_status hils_decode_fwd_paged(const hils_params *p, const void *q,
                                           const void *k_pages, const void *v_pages,
                                           int64_t num_pages, const int32_t *page_table,
                                           int max_pages_per_seq, const void *lmk_k,
                                           int32_t *sel_idx, float *chunk_w, float *lse_lmk,
                                           void *out, float *lse, void *ws, size_t ws_bytes,
                                           void *stream) {
  hils_status s = check_params(p);
  if (s != HILS_OK) return s;
  NEED(q);
  NEED(k_pages);
  NEED(v_pages);
  NEED(page_table);
  const int pages_needed = (p->L + p->chunk - 1) / p->chunk;
  if (max_pages_per_seq < pages_needed)
    return fail(HILS_ERR_INVALID_ARG, "max_pages_per_seq %d below the %d pages of N=%d",
                max_pages_per_seq, pages_needed, p->L);
  if (num_pages < 1) return fail(HILS_ERR_INVALID_ARG, "num_pages must be >= 1");
  if ((int64_t)p->B * max_pages_per_seq >= (int64_t)1 << 31)
    return fail(HILS_ERR_UNSUPPORTED, "B * max_pages_per_seq must be below 2^31");
  return decode_impl(p, q, k_pages, v_pages,
                     hils::PagedKV{page_table, max_pages_per_seq, (long long)num_pages}, lmk_k,
                     sel_idx, chunk_w, lse_lmk, out, lse, ws, ws_bytes, stream);
}

HILS_API size_t hils_qcal_workspace_size(const hils_params *p, int r) {
  if (check_params(p) != HILS_OK || r < 1 || r > hils::kMaxQcalRank) return 0;
  return kDebugWs + (((size_t)p->B * p->L * r * sizeof(float) + 255) & ~size_t(255));
}

HILS_API hils_status hils_qcal_query(const hils_params *p, const void *q, const void *h,
                                     const void *w_down, const void *w_up, int D, int r,
                                     void *q_cal, void *ws, size_t ws_bytes, void *stream) {
  hils_status s = check_params(p);
  if (s != HILS_OK) return s;
  NEED(q);
  NEED(h);
  NEED(w_down);
  NEED(w_up);
  NEED(q_cal);
  if (D < 1) return fail(HILS_ERR_INVALID_ARG, "D=%d must be >= 1", D);
  if (r < 1 || r > hils::kMaxQcalRank)
    return fail(HILS_ERR_UNSUPPORTED, "r=%d (supported: 1..%d)", r, hils::kMaxQcalRank);
  if ((int64_t)p->B * p->L * D >= (int64_t)1 << 40)
    return fail(HILS_ERR_UNSUPPORTED, "B*L*D too large");
  const size_t need = hils_qcal_workspace_size(p, r);
  if (!ws || ws_bytes < need)
    return fail(HILS_ERR_WORKSPACE, "Q-Cal needs %zu bytes of workspace, got %zu", need, ws_bytes);
  NEED(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float *z = reinterpret_cast<float *>(static_cast<unsigned char *>(ws) + kDebugWs);
  int n = 0;
  cudaError_t e = hils::qcal_query(p->dtype == HILS_BF16, p->B, p->Hq, p->L, p->d, D, r, q, h,
                                   w_down, w_up, q_cal, z, st, &n);
  g_launches += n;
  if (e != cudaSuccess) return cuda_fail(e, "Q-Cal launch");
  return HILS_OK;
}

HILS_API hils_status hils_prefill_qcal(const hils_params *p, const void *q, const void *k,
                                       const void *v, const void *lmk_k, const void *h,
                                       const void *w_down, const void *w_up, int D, int r,
                                       void *q_cal, int32_t *sel_idx, float *chunk_w,
                                       float *lse_lmk, void *out, float *lse, void *ws,
                                       size_t ws_bytes, void *stream) {
  hils_status s = hils_qcal_query(p, q, h, w_down, w_up, D, r, q_cal, ws, ws_bytes, stream);
  if (s != HILS_OK) return s;
  s = hils_select(p, q_cal, lmk_k, sel_idx, chunk_w, lse_lmk, ws, ws_bytes, stream);
  if (s != HILS_OK) return s;
  return hils_attn_fwd(p, q, k, v, sel_idx, chunk_w, out, lse, nullptr, ws, ws_bytes, stream);
}

HILS_API hils_status hils_hope(void *x, int dtype, int B, int H, int L, int d, int pos0,
                               int n_rope_pairs, double base, void *stream) {
  NEED(x);
  if (dtype != HILS_F32 && dtype != HILS_BF16) return fail(HILS_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (B < 1 || H < 1 || L < 1) return fail(HILS_ERR_INVALID_ARG, "B, H and L must be >= 1");
  if (d != 64 && d != 128) return fail(HILS_ERR_UNSUPPORTED, "d=%d (supported: 64, 128)", d);
  if (n_rope_pairs < 0 || n_rope_pairs > d / 2)
    return fail(HILS_ERR_INVALID_ARG, "n_rope_pairs=%d outside [0, d/2]", n_rope_pairs);
  if (pos0 < 0 || (int64_t)pos0 + L - 1 >= (int64_t)1 << 31)
    return fail(HILS_ERR_INVALID_ARG, "positions pos0 .. pos0+L-1 must lie in [0, 2^31)");
  if (!std::isfinite(base) || !(base > 1.0)) return fail(HILS_ERR_INVALID_ARG, "base must be finite and > 1");
  if ((int64_t)B * H > (1 << 16) - 1) return fail(HILS_ERR_UNSUPPORTED, "B*H above 65535");
  int n = 0;
  cudaError_t e = hils::hope_apply(x, dtype == HILS_BF16, B * H, L, d, pos0, n_rope_pairs, base,
                                   static_cast<cudaStream_t>(stream), &n);
  g_launches += n;
  if (e != cudaSuccess) return cuda_fail(e, "hope launch");
  return HILS_OK;
}

HILS_API hils_status hils_prefill_hope(const hils_params *p, const void *q, const void *k,
                                       const void *v, const void *lmk_k, int pos0,
                                       int n_rope_pairs, double base, int32_t *sel_idx,
                                       float *chunk_w, float *lse_lmk, void *out, float *lse,
                                       void *ws, size_t ws_bytes, void *stream) {
  hils_status s = check_params(p);
  if (s != HILS_OK) return s;
  if (p->dtype != HILS_BF16)
    return fail(HILS_ERR_UNSUPPORTED,
                "the fused HoPE prefill runs on the bf16 tensor-core path; rotate fp32 queries "
                "with hils_hope and call hils_prefill");
  if (n_rope_pairs < 0 || n_rope_pairs > p->d / 2)
    return fail(HILS_ERR_INVALID_ARG, "n_rope_pairs=%d outside [0, d/2]", n_rope_pairs);
  if (pos0 < 0 || (int64_t)pos0 + p->L - 1 >= (int64_t)1 << 31)
    return fail(HILS_ERR_INVALID_ARG, "positions pos0 .. pos0+L-1 must lie in [0, 2^31)");
  if (!std::isfinite(base) || !(base > 1.0)) return fail(HILS_ERR_INVALID_ARG, "base must be finite and > 1");
  NEED(q);
  NEED(k);
  NEED(v);
  NEED(sel_idx);
  NEED(chunk_w);
  MAYBE(lse_lmk);
  NEED(out);
  NEED(lse);
  if (p->L >= p->chunk) NEED(lmk_k);
  const hils::HopeParams hp = hils::hope_params(p->d, n_rope_pairs, pos0, base);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t *err = nullptr;
  if ((s = debug_begin(p, ws, ws_bytes, &err, st)) != HILS_OK) return s;
  const hils::RowSpec rs = prefill_rows(p);
  if ((s = do_select(p, rs, q, lmk_k, sel_idx, chunk_w, lse_lmk, err, st, hp)) != HILS_OK) return s;
  if ((s = do_attn(p, rs, q, k, v, sel_idx, chunk_w, out, lse, nullptr, err, st, hp)) != HILS_OK)
    return s;
  return debug_end(err, st);
}

HILS_API size_t hils_attn_bwd_workspace_size(const hils_params *p) {
  if (check_params(p) != HILS_OK) return 0;
  return hils::bwd_workspace_bytes(
      hils::bwd_spec(p->B, p->Hq, p->Hkv, p->L, p->d, p->topk, p->scale));
}

HILS_API hils_status hils_attn_bwd(const hils_params *p, const void *q, const void *k,
                                   const void *v, const void *lmk_k, const int32_t *sel_idx,
                                   const float *chunk_w, const float *lse, const void *dout,
                                   const float *dlse, float *dq, float *dk, float *dv,
                                   float *dlmk, void *ws, size_t ws_bytes, void *stream) {
  hils_status s = check_params(p);
  if (s != HILS_OK) return s;
  NEED(q);
  NEED(k);
  NEED(v);
  NEED(sel_idx);
  NEED(chunk_w);
  NEED(lse);
  NEED(dout);
  MAYBE(dlse);
  NEED(dq);
  NEED(dk);
  NEED(dv);
  if (p->L >= p->chunk) {
    NEED(lmk_k);
    NEED(dlmk);
  }
  if ((int64_t)p->B * p->Hq * p->L * p->topk >= (int64_t)1 << 31)
    return fail(HILS_ERR_UNSUPPORTED, "B*Hq*L*topk must be below 2^31 for the backward pass");
  const hils::BwdSpec bs = hils::bwd_spec(p->B, p->Hq, p->Hkv, p->L, p->d, p->topk, p->scale);
  const size_t need = hils::bwd_workspace_bytes(bs);
  if (!ws || ws_bytes < need)
    return fail(HILS_ERR_WORKSPACE, "backward needs %zu bytes of workspace, got %zu", need, ws_bytes);
  NEED(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t *err = nullptr;
  if ((s = debug_begin(p, ws, ws_bytes, &err, st)) != HILS_OK) return s;
  int n = 0;
  cudaError_t e = hils::bwd_run(bs, p->dtype == HILS_BF16, q, k, v, lmk_k, sel_idx, chunk_w, lse,
                                dout, dlse, dq, dk, dv, dlmk, ws, err, st, &n);
  g_launches += n;
  if (e != cudaSuccess) return cuda_fail(e, "backward launch");
  return debug_end(err, st);
}

HILS_API void hils_test_set_wait_limit(uint64_t ns, int withhold) {
  g_test_wait_ns.store(ns);
  g_test_withhold.store(withhold ? 1 : 0);
}

HILS_API int hils_hope_rope_pairs(int d, double base, double train_len) {
  // pairs i (rotate-half) whose wavelength 2 pi base^(2i/d) fits the window;
  // the wavelength grows with i, so they are the first ones
  if (d < 2 || !(base > 1.0) || !std::isfinite(base) || std::isnan(train_len)) return -1;
  const double two_pi = 6.283185307179586;
  int n = 0;
  while (n < d / 2 && two_pi * std::pow(base, 2.0 * n / d) <= train_len) ++n;
  return n;
}

HILS_API const char *hils_status_string(hils_status s) {
  switch (s) {
    case HILS_OK: return "ok";
    case HILS_ERR_INVALID_ARG: return "invalid argument";
    case HILS_ERR_UNSUPPORTED: return "unsupported configuration";
    case HILS_ERR_WORKSPACE: return "workspace too small";
    case HILS_ERR_CUDA: return "CUDA error";
    case HILS_ERR_DEVICE_CHECK: return "device-side check failed";
    case HILS_ERR_TIMEOUT: return "bounded device wait timed out";
  }
  return "unknown status";
}

HILS_API const char *hils_last_error(void) { return g_msg; }

extern "C" void hils_internal_set_error(const char *msg) { fail(HILS_ERR_INVALID_ARG, "%s", msg); }

HILS_API int64_t hils_launch_count(void) { return g_launches.load(); }
