// C ABI front end of libvqlinear: argument validation, handle management, the
// per-forward plan and kernel dispatch.  Every argument problem is caught here,
// on the host, before anything is enqueued.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "internal.h"
#include "tools.h"
#include "vqlinear.h"
#include "vqlinear_tools.h"

#define VQ_API extern "C" __attribute__((visibility("default")))

namespace vq {
void plan_gemv(const vq_linear_desc& d, const DeviceInfo& dev, int M, Plan* p);
bool plan_lut(const vq_linear_desc& d, const DeviceInfo& dev, int M, Plan* p);
bool plan_tc(const vq_linear_desc& d, const DeviceInfo& dev, int M, Plan* p);
bool plan_vq16(const vq_linear_desc& d, const DeviceInfo& dev, int M, Plan* p);
}  // namespace vq

struct vq_linear_s {
  vq_linear_desc d;
  vq::DeviceInfo dev;
  int path;
  float* scratch;
  size_t scratch_bytes;
  uint32_t* tickets;  // completion counters, zeroed at create, left zero by every forward
  int num_tickets;
  uint32_t* sync;     // the table kernel's cross-CTA words (zeroed at create)
  int num_sync;
  uint32_t* err;      // device word, set by bounded waits that gave up
  int sm_budget;      // CTAs of the table kernel (0: every SM)
  void* xrot;         // rotated-x buffer [max_M][K] (desc.rht == 1), for the unfused rotated forward
  float* corr_y;      // the sparse correction's x . C^T, fp32 [max_M][N] (desc.corr == 1)
};

namespace {

thread_local std::string t_err;

vq_status fail(vq_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_err = buf;
  return st;
}

vq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(VQ_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

vq_status check_ptr(const void* p, const char* name) {
  if (p == nullptr) return fail(VQ_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(p)) return fail(VQ_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return VQ_OK;
}

vq_status validate_desc(const vq_linear_desc* d) {
  if (d == nullptr) return fail(VQ_ERR_INVALID_ARG, "desc is NULL");
  if (d->N <= 0 || d->K <= 0) return fail(VQ_ERR_INVALID_ARG, "N=%d and K=%d must be positive", d->N, d->K);
  if (d->K % 16 != 0) return fail(VQ_ERR_INVALID_ARG, "K=%d is not a multiple of 16 (two groups of 8)", d->K);
  if (d->K % 64 != 0) return fail(VQ_ERR_UNSUPPORTED, "K=%d: this library needs K to be a multiple of 64", d->K);
  if (d->N > (1 << 24) || d->K > (1 << 24))
    return fail(VQ_ERR_UNSUPPORTED, "N=%d / K=%d exceed the supported 2^24", d->N, d->K);
  if (d->fmt != VQ_FMT_RVQ12 && d->fmt != VQ_FMT_RVQ12_4 && d->fmt != VQ_FMT_VQ16 && d->fmt != VQ_FMT_VQ16_RVQ)
    return fail(VQ_ERR_INVALID_ARG, "fmt=%d is not a VQ_FMT_* value", d->fmt);
  if (d->fmt == VQ_FMT_VQ16_RVQ) {
    if (d->n16 < 1 || d->n16 > 4 || d->n8 < 0 || d->n8 > 1 || d->n16 + d->n8 > 4)
      return fail(VQ_ERR_INVALID_ARG, "n16=%d, n8=%d: need 1 <= n16, 0 <= n8 <= 1, n16 + n8 <= 4", d->n16, d->n8);
    for (int t = 0; t < d->n16 + d->n8 - 1; ++t)
      if (!std::isfinite(d->mult[t])) return fail(VQ_ERR_INVALID_ARG, "mult[%d] is not finite", t);
  }
  if (d->scale_group <= 0 || d->scale_group % 8 != 0 || d->K % d->scale_group != 0)
    return fail(VQ_ERR_INVALID_ARG, "scale_group=%d must be a positive multiple of 8 dividing K", d->scale_group);
  if (d->scale_group != 64 && d->scale_group != d->K)
    return fail(VQ_ERR_UNSUPPORTED, "scale_group=%d: only 64 or K (per row) are implemented", d->scale_group);
  if (d->act_dtype != VQ_F16 && d->act_dtype != VQ_BF16)
    return fail(VQ_ERR_INVALID_ARG, "act_dtype=%d is not VQ_F16 or VQ_BF16", d->act_dtype);
  if (d->max_M <= 0 || d->max_M > (1 << 20))
    return fail(VQ_ERR_INVALID_ARG, "max_M=%d must be in [1, 2^20]", d->max_M);
  if (d->corr != 0 && d->corr != 1) return fail(VQ_ERR_INVALID_ARG, "corr=%d must be 0 or 1", d->corr);
  if (d->corr && d->fmt == VQ_FMT_VQ16_RVQ)
    return fail(VQ_ERR_UNSUPPORTED, "the sparse correction is defined for the 12-bit and 16-bit formats only");
  return VQ_OK;
}

vq_status validate_planes(const vq_linear_desc& d, const vq_planes* p) {
  if (p == nullptr) return fail(VQ_ERR_INVALID_ARG, "planes is NULL");
  vq_status st;
  if (d.fmt == VQ_FMT_VQ16 || d.fmt == VQ_FMT_VQ16_RVQ) {
    if ((st = check_ptr(p->idx16, "planes->idx16"))) return st;
    if (d.fmt == VQ_FMT_VQ16_RVQ && d.n8 && (st = check_ptr(p->idx8, "planes->idx8"))) return st;
  } else {
    if ((st = check_ptr(p->lo, "planes->lo"))) return st;
    if ((st = check_ptr(p->hi4, "planes->hi4"))) return st;
    if (d.fmt == VQ_FMT_RVQ12_4 && (st = check_ptr(p->s2, "planes->s2"))) return st;
  }
  if (d.corr) {
    if ((st = check_ptr(p->corr_rows, "planes->corr_rows"))) return st;
    if (p->corr_cols && !aligned16(p->corr_cols)) return fail(VQ_ERR_INVALID_ARG, "planes->corr_cols is not 16-byte aligned");
    if (p->corr_vals && !aligned16(p->corr_vals)) return fail(VQ_ERR_INVALID_ARG, "planes->corr_vals is not 16-byte aligned");
    if ((p->corr_cols == nullptr) != (p->corr_vals == nullptr))
      return fail(VQ_ERR_INVALID_ARG, "planes->corr_cols and corr_vals must both be given (or both NULL: no entries)");
  } else if (p->corr_rows || p->corr_cols || p->corr_vals) {
    return fail(VQ_ERR_INVALID_ARG, "planes carry a sparse correction but the handle was created with corr = 0");
  }
  return VQ_OK;
}

vq_status validate_codebooks(const vq_linear_desc& d, const vq_codebooks* cb, const void* scales) {
  if (cb == nullptr) return fail(VQ_ERR_INVALID_ARG, "codebooks is NULL");
  vq_status st;
  if ((st = check_ptr(cb->cb1, "codebooks->cb1"))) return st;
  if (d.fmt == VQ_FMT_RVQ12_4 && (st = check_ptr(cb->cb2, "codebooks->cb2"))) return st;
  if (d.fmt == VQ_FMT_VQ16_RVQ) {
    for (int t = 0; t < d.n16 - 1; ++t)
      if ((st = check_ptr(cb->cbr[t], "codebooks->cbr[t]"))) return st;
    if (d.n8 && (st = check_ptr(cb->cb8, "codebooks->cb8"))) return st;
  }
  if ((st = check_ptr(scales, "scales"))) return st;
  return VQ_OK;
}

vq_status check_device(const vq_linear_s* h) {
  int cur = -1;
  cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (cur != h->dev.device)
    return fail(VQ_ERR_INVALID_ARG, "current device %d differs from the handle's device %d", cur, h->dev.device);
  return VQ_OK;
}

vq::LayerArgs make_args(const vq_linear_desc& d, const vq_planes* p, const vq_codebooks* cb, const void* scales) {
  vq::LayerArgs a{};
  a.lo = p ? p->lo : nullptr;
  a.hi4 = p ? p->hi4 : nullptr;
  a.s2 = p ? p->s2 : nullptr;
  a.idx16 = p ? p->idx16 : nullptr;
  if (p && d.corr) {
    a.corr_rows = p->corr_rows;
    a.corr_cols = p->corr_cols;
    a.corr_vals = p->corr_vals;
  }
  a.cb1 = cb ? static_cast<const uint16_t*>(cb->cb1) : nullptr;
  a.cb2 = cb ? static_cast<const uint16_t*>(cb->cb2) : nullptr;
  a.scales = static_cast<const uint16_t*>(scales);
  a.N = d.N;
  a.K = d.K;
  a.fmt = d.fmt;
  a.scale_group = d.scale_group;
  a.act = d.act_dtype;
  a.n16 = 1;
  a.n8 = 0;
  if (d.fmt == VQ_FMT_VQ16_RVQ) {  // only the entries the stage counts use are read
    a.n16 = d.n16;
    a.n8 = d.n8;
    a.idx8 = (p && d.n8) ? p->idx8 : nullptr;
    for (int t = 0; t < 3; ++t) {
      a.cbr[t] = (cb && t < d.n16 - 1) ? static_cast<const uint16_t*>(cb->cbr[t]) : nullptr;
      a.mult[t] = t < d.n16 + d.n8 - 1 ? d.mult[t] : 0.f;
    }
    a.cb8 = (cb && d.n8) ? static_cast<const uint16_t*>(cb->cb8) : nullptr;
  }
  return a;
}

}  // namespace

namespace vq {

bool plan_forward(const vq_linear_desc& d, const DeviceInfo& dev, int M, int forced_path, Plan* out) {
  int path = forced_path;
  if (path == VQ_PATH_AUTO) {
    // Measured on B200: from M = 2 the tensor-core path decodes large layers
    // faster than the warp-MMA GEMV; on small layers both are launch-bound.
    const bool large = (int64_t)d.N * d.K >= (int64_t(1) << 22);
    path = (M == 1) ? VQ_PATH_LUT : ((M <= 16 && !large) ? VQ_PATH_GEMV : VQ_PATH_TC);
    // 16-bit indices, up to 4 tokens: the gather kernel where it applies (measured on
    // B200, 4096 x 4096: faster than the tensor-core path up to M = 4, slower at 8)
    if ((d.fmt == VQ_FMT_VQ16 || d.fmt == VQ_FMT_VQ16_RVQ) && M <= 4 && plan_vq16(d, dev, M, out)) return true;
  }
  switch (path) {
    case VQ_PATH_GATHER:
      return plan_vq16(d, dev, M, out);
    case VQ_PATH_LUT:
      if (plan_lut(d, dev, M, out)) return true;
      if (forced_path != VQ_PATH_AUTO) return false;
      path = VQ_PATH_GEMV;
      [[fallthrough]];
    case VQ_PATH_GEMV:
      if (M < 1 || M > 16) {
        if (forced_path != VQ_PATH_AUTO) return false;
        return plan_tc(d, dev, M, out);
      }
      plan_gemv(d, dev, M, out);
      return true;
    case VQ_PATH_TC:
      if (plan_tc(d, dev, M, out)) return true;
      if (forced_path != VQ_PATH_AUTO || M > 16) return false;
      plan_gemv(d, dev, M, out);
      return true;
    default:
      return false;
  }
}

}  // namespace vq

VQ_API int32_t vq_abi_version(void) { return 3; }

VQ_API const char* vq_last_error(void) { return t_err.c_str(); }

VQ_API vq_status vq_linear_create(const vq_linear_desc* desc, vq_linear_t* out) {
  if (out == nullptr) return fail(VQ_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  vq_status st = validate_desc(desc);
  if (st) return st;
  vq::DeviceInfo dev{};
  cudaError_t e = cudaGetDevice(&dev.device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev.device);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev.device);
  if (major != 10 || minor != 0)
    return fail(VQ_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a only", dev.device,
                major, minor);
  cudaDeviceGetAttribute(&dev.num_sms, cudaDevAttrMultiProcessorCount, dev.device);
  cudaDeviceGetAttribute(&dev.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev.device);

  // Scratch: the largest any path may need for any M <= max_M.
  size_t need = 0;
  int tickets = 0, sync_words = 0;
  for (int M = 1; M <= desc->max_M; ++M) {
    const int paths[4] = {VQ_PATH_LUT, VQ_PATH_GEMV, VQ_PATH_TC, VQ_PATH_GATHER};
    for (int pth : paths) {
      vq::Plan p{};
      if (!vq::plan_forward(*desc, dev, M, pth, &p)) continue;
      if (p.scratch_bytes > need) need = p.scratch_bytes;
      if (p.tickets > tickets) tickets = p.tickets;
      if (p.sync_words > sync_words) sync_words = p.sync_words;
    }
  }
  // Test hook: VQ_TEST_FAIL_ALLOC=1 makes the device allocations fail, so callers'
  // handling of VQ_ERR_NOMEM can be tested without exhausting a shared GPU.
  const char* fail_alloc = getenv("VQ_TEST_FAIL_ALLOC");
  if (fail_alloc && fail_alloc[0] == '1')
    return fail(VQ_ERR_NOMEM, "device allocation refused (VQ_TEST_FAIL_ALLOC=1)");
  vq_linear_s* h = new (std::nothrow) vq_linear_s{};
  if (!h) return fail(VQ_ERR_NOMEM, "host allocation of the handle failed");
  h->d = *desc;
  h->dev = dev;
  h->path = VQ_PATH_AUTO;
  h->scratch_bytes = need;
  if (need) {
    e = cudaMalloc(&h->scratch, need);
    if (e != cudaSuccess) {
      delete h;
      cudaGetLastError();
      return fail(VQ_ERR_NOMEM, "cudaMalloc of %zu scratch bytes failed: %s", need, cudaGetErrorString(e));
    }
  }
  if (desc->rht) {
    e = cudaMalloc(&h->xrot, (size_t)desc->max_M * desc->K * 2);
    if (e != cudaSuccess) {
      cudaFree(h->scratch);
      delete h;
      cudaGetLastError();
      return fail(VQ_ERR_NOMEM, "cudaMalloc of the %d x %d rotation buffer failed: %s", desc->max_M, desc->K,
                  cudaGetErrorString(e));
    }
  }
  if (desc->corr) {
    e = cudaMalloc(&h->corr_y, (size_t)desc->max_M * desc->N * sizeof(float));
    if (e != cudaSuccess) {
      cudaFree(h->scratch);
      cudaFree(h->xrot);
      delete h;
      cudaGetLastError();
      return fail(VQ_ERR_NOMEM, "cudaMalloc of the %d x %d correction buffer failed: %s", desc->max_M, desc->N,
                  cudaGetErrorString(e));
    }
  }
  h->num_tickets = tickets;
  h->num_sync = sync_words;
  // words: [0] error flag, [1] pad, then the tickets, then the table kernel's sync words
  const size_t small = sizeof(uint32_t) * (2 + (size_t)tickets + (size_t)sync_words);
  uint32_t* words = nullptr;
  e = cudaMalloc(&words, small);
  if (e == cudaSuccess) e = cudaMemset(words, 0, small);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();  // the zeroing is complete before any forward
  h->err = words;
  h->tickets = (words && tickets) ? words + 2 : nullptr;
  h->sync = (words && sync_words) ? words + 2 + tickets : nullptr;
  if (e != cudaSuccess) {
    cudaFree(h->scratch);
    cudaFree(h->xrot);
    cudaFree(h->corr_y);
    cudaFree(words);
    delete h;
    cudaGetLastError();
    return fail(VQ_ERR_NOMEM, "cudaMalloc of the error word failed: %s", cudaGetErrorString(e));
  }
  *out = h;
  return VQ_OK;
}

VQ_API vq_status vq_linear_destroy(vq_linear_t h) {
  if (h == nullptr) return VQ_OK;
  cudaError_t e1 = cudaSuccess, e2 = cudaSuccess;
  // Wait for the handle's device to finish all enqueued work (a forward still in
  // flight may read the scratch or the counters freed below), on that device.
  int prev = -1;
  e1 = cudaGetDevice(&prev);
  if (e1 == cudaSuccess && prev != h->dev.device) e1 = cudaSetDevice(h->dev.device);
  if (e1 == cudaSuccess) e1 = cudaDeviceSynchronize();
  if (e1 != cudaSuccess) {
    if (prev >= 0 && prev != h->dev.device) cudaSetDevice(prev);
    delete h;  // the device memory is unreachable now; report the error
    return cuda_fail(e1, "vq_linear_destroy: synchronising the handle's device");
  }
  if (h->scratch) e1 = cudaFree(h->scratch);
  if (h->xrot && e1 == cudaSuccess) e1 = cudaFree(h->xrot);
  if (h->corr_y && e1 == cudaSuccess) e1 = cudaFree(h->corr_y);
  if (h->err) e2 = cudaFree(h->err);  // also frees the tickets and sync words (one allocation)
  if (prev >= 0 && prev != h->dev.device) cudaSetDevice(prev);
  delete h;
  if (e1 != cudaSuccess) return cuda_fail(e1, "cudaFree(scratch)");
  if (e2 != cudaSuccess) return cuda_fail(e2, "cudaFree(err)");
  return VQ_OK;
}

VQ_API vq_status vq_linear_set_path(vq_linear_t h, int32_t path) {
  if (h == nullptr) return fail(VQ_ERR_INVALID_ARG, "handle is NULL");
  if (path < VQ_PATH_AUTO || path > VQ_PATH_GATHER) return fail(VQ_ERR_INVALID_ARG, "path=%d is not a VQ_PATH_*", path);
  h->path = path;
  return VQ_OK;
}

VQ_API vq_status vq_linear_set_sm_budget(vq_linear_t h, int32_t sms) {
  if (h == nullptr) return fail(VQ_ERR_INVALID_ARG, "handle is NULL");
  if (sms < 0 || sms > h->dev.num_sms)
    return fail(VQ_ERR_INVALID_ARG, "sms=%d outside [0, %d] (0 = every SM)", sms, h->dev.num_sms);
  h->sm_budget = sms;
  return VQ_OK;
}

VQ_API int32_t vq_linear_launches(vq_linear_t h, int32_t M) {
  if (h == nullptr || M < 0 || M > h->d.max_M) return -1;
  if (M == 0) return 0;
  vq::Plan p{};
  if (!vq::plan_forward(h->d, h->dev, M, h->path, &p)) return -1;
  return p.launches + (h->d.corr ? 1 : 0);  // the sparse correction's kernel
}

VQ_API vq_status vq_linear_plan(vq_linear_t h, int32_t M, vq_plan_info* out) {
  if (h == nullptr || out == nullptr) return fail(VQ_ERR_INVALID_ARG, "handle or out is NULL");
  if (M < 1 || M > h->d.max_M) return fail(VQ_ERR_INVALID_ARG, "M=%d outside [1, max_M=%d]", M, h->d.max_M);
  vq::Plan p{};
  if (!vq::plan_forward(h->d, h->dev, M, h->path, &p))
    return fail(VQ_ERR_UNSUPPORTED, "path %d cannot run M=%d for this layer", h->path, M);
  if ((p.path == VQ_PATH_LUT || p.path == VQ_PATH_GATHER) && h->sm_budget > 0 && p.grid > h->sm_budget)
    p.ctas = h->sm_budget;  // as the forward clamps its grid
  out->path = p.path;
  out->launches = p.launches + (h->d.corr ? 1 : 0);
  out->ctas = p.ctas;
  out->splits = p.splits;
  return VQ_OK;
}

VQ_API vq_status vq_plan_for_device(const vq_linear_desc* desc, int32_t M, int32_t path, int32_t num_sms,
                                    int32_t smem_optin, vq_plan_info* out) {
  vq_status st = validate_desc(desc);
  if (st) return st;
  if (out == nullptr) return fail(VQ_ERR_INVALID_ARG, "out is NULL");
  if (M < 1 || M > desc->max_M) return fail(VQ_ERR_INVALID_ARG, "M=%d outside [1, max_M=%d]", M, desc->max_M);
  if (num_sms < 1 || smem_optin < 0)
    return fail(VQ_ERR_INVALID_ARG, "num_sms=%d and smem_optin=%d: need num_sms >= 1, smem_optin >= 0", num_sms,
                smem_optin);
  if (path < VQ_PATH_AUTO || path > VQ_PATH_GATHER) return fail(VQ_ERR_INVALID_ARG, "path=%d is not a VQ_PATH_*", path);
  vq::DeviceInfo dev{};
  dev.device = -1;
  dev.num_sms = num_sms;
  dev.smem_optin = smem_optin;
  vq::Plan p{};
  if (!vq::plan_forward(*desc, dev, M, path, &p))
    return fail(VQ_ERR_UNSUPPORTED, "path %d cannot run M=%d for this layer on this device", path, M);
  out->path = p.path;
  out->launches = p.launches + (desc->corr ? 1 : 0);
  out->ctas = p.ctas;
  out->splits = p.splits;
  return VQ_OK;
}

VQ_API vq_status vq_linear_forward(vq_linear_t h, const void* x, const vq_planes* planes,
                                   const vq_codebooks* codebooks, const void* scales, void* y, int32_t M,
                                   int32_t N, int32_t K, void* stream) {
  if (h == nullptr) return fail(VQ_ERR_INVALID_ARG, "handle is NULL");
  const vq_linear_desc& d = h->d;
  if (N != d.N || K != d.K)
    return fail(VQ_ERR_INVALID_ARG, "N=%d, K=%d do not match the handle's N=%d, K=%d", N, K, d.N, d.K);
  if (M < 0 || M > d.max_M) return fail(VQ_ERR_INVALID_ARG, "M=%d outside [0, max_M=%d]", M, d.max_M);
  vq_status st;
  if ((st = check_ptr(x, "x")) || (st = check_ptr(y, "y")) || (st = validate_planes(d, planes)) ||
      (st = validate_codebooks(d, codebooks, scales)))
    return st;
  if (x == y) return fail(VQ_ERR_INVALID_ARG, "y must not alias x");
  if (M == 0) return VQ_OK;
  if ((st = check_device(h))) return st;
  vq::Plan p{};
  if (!vq::plan_forward(d, h->dev, M, h->path, &p))
    return fail(VQ_ERR_UNSUPPORTED, "path %d cannot run M=%d", h->path, M);
  if ((p.path == VQ_PATH_LUT || p.path == VQ_PATH_GATHER) && h->sm_budget > 0 && p.grid > h->sm_budget)
    p.grid = h->sm_budget;
  if (p.scratch_bytes > h->scratch_bytes || p.tickets > h->num_tickets || p.sync_words > h->num_sync)
    return fail(VQ_ERR_UNSUPPORTED, "plan needs %zu scratch bytes / %d tickets / %d sync words, handle has %zu / %d / %d",
                p.scratch_bytes, p.tickets, p.sync_words, h->scratch_bytes, h->num_tickets, h->num_sync);
  vq::LayerArgs a = make_args(d, planes, codebooks, scales);
  a.x = x;
  a.y = y;
  a.M = M;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (d.corr) {  // x . C^T first, in fp32; the forward kernel adds it before rounding
    e = vq::launch_corr(a, h->corr_y, s);
    if (e != cudaSuccess) return cuda_fail(e, "vq_linear_forward correction launch");
    a.addend = h->corr_y;
  }
  switch (p.path) {
    case VQ_PATH_LUT: e = vq::launch_lut(a, p, h->scratch, h->sync, h->err, s); break;  // p.grid CTAs
    case VQ_PATH_GATHER: e = vq::launch_vq16(a, p, nullptr, s); break;
    case VQ_PATH_TC: e = vq::launch_tc(a, p, h->scratch, h->tickets, h->err, s); break;
    default: e = vq::launch_gemv(a, p, h->scratch, h->tickets, s); break;
  }
  if (e != cudaSuccess) return cuda_fail(e, "vq_linear_forward launch");
  return VQ_OK;
}

VQ_API vq_status vq_linear_forward_rotated(vq_linear_t h, const void* x, const int8_t* signs, const vq_planes* planes,
                                           const vq_codebooks* codebooks, const void* scales, void* y, int32_t M,
                                           int32_t N, int32_t K, void* stream) {
  if (h == nullptr) return fail(VQ_ERR_INVALID_ARG, "handle is NULL");
  const vq_linear_desc& d = h->d;
  if (N != d.N || K != d.K)
    return fail(VQ_ERR_INVALID_ARG, "N=%d, K=%d do not match the handle's N=%d, K=%d", N, K, d.N, d.K);
  if (K < 64 || K > 32768 || K % 64 != 0)
    return fail(VQ_ERR_INVALID_ARG, "K=%d: the rotation needs a multiple of 64 in [64, 32768]", K);
  if (M < 0 || M > d.max_M) return fail(VQ_ERR_INVALID_ARG, "M=%d outside [0, max_M=%d]", M, d.max_M);
  vq_status st;
  if ((st = check_ptr(signs, "signs")) || (st = check_ptr(x, "x")) || (st = check_ptr(y, "y")) || (st = validate_planes(d, planes)) ||
      (st = validate_codebooks(d, codebooks, scales)))
    return st;
  if (x == y) return fail(VQ_ERR_INVALID_ARG, "y must not alias x");
  if (M == 0) return VQ_OK;
  if ((st = check_device(h))) return st;
  vq::Plan p{};
  if (!vq::plan_forward(d, h->dev, M, h->path, &p))
    return fail(VQ_ERR_UNSUPPORTED, "path %d cannot run M=%d", h->path, M);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Where the forward runs the 16-bit gather kernel (automatically up to M = 4, or
  // forced up to M = 8) that kernel rotates x itself: one launch, no rotated copy of
  // x in memory.  (A sparse correction needs the rotated x too: that layer takes the
  // route below.)
  if (p.path == VQ_PATH_GATHER && !d.corr) {
    if (h->sm_budget > 0 && p.grid > h->sm_budget) p.grid = h->sm_budget;
    if (p.scratch_bytes > h->scratch_bytes)
      return fail(VQ_ERR_UNSUPPORTED, "plan needs %zu scratch bytes, handle has %zu", p.scratch_bytes,
                  h->scratch_bytes);
    vq::LayerArgs a = make_args(d, planes, codebooks, scales);
    a.x = x;
    a.y = y;
    a.M = M;
    cudaError_t e = vq::launch_vq16(a, p, signs, s);
    if (e != cudaSuccess) return cuda_fail(e, "vq_linear_forward_rotated launch");
    return VQ_OK;
  }
  if (h->xrot == nullptr)
    return fail(VQ_ERR_INVALID_ARG,
                "this shape's rotation is not fused and the handle has no rotation buffer (create it with rht = 1)");
  cudaError_t e = vq::launch_rht(x, h->xrot, signs, M, K, d.act_dtype, s);
  if (e != cudaSuccess) return cuda_fail(e, "vq_linear_forward_rotated rotation launch");
  return vq_linear_forward(h, h->xrot, planes, codebooks, scales, y, M, N, K, stream);
}

VQ_API vq_status vq_rht_apply(const void* x, void* x_out, const int8_t* signs, int32_t M, int32_t K, int32_t dtype,
                              void* stream) {
  if (K < 64 || K > 32768 || K % 64 != 0)
    return fail(VQ_ERR_INVALID_ARG, "K=%d must be a multiple of 64 in [64, 32768]", K);
  if (M < 0) return fail(VQ_ERR_INVALID_ARG, "M=%d is negative", M);
  if (dtype != VQ_F16 && dtype != VQ_BF16) return fail(VQ_ERR_INVALID_ARG, "dtype=%d", dtype);
  vq_status st;
  if ((st = check_ptr(x, "x")) || (st = check_ptr(x_out, "x_out")) || (st = check_ptr(signs, "signs"))) return st;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(x), b0 = reinterpret_cast<uintptr_t>(x_out);
  const uintptr_t bytes = (uintptr_t)M * K * 2;
  if (a0 != b0 && a0 < b0 + bytes && b0 < a0 + bytes)
    return fail(VQ_ERR_INVALID_ARG, "x_out partially overlaps x");
  if (M == 0) return VQ_OK;
  cudaError_t e = vq::launch_rht(x, x_out, signs, M, K, dtype, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "vq_rht_apply launch");
  return VQ_OK;
}

VQ_API vq_status vq_rht_apply_output(const void* y, void* y_out, const int8_t* signs, int32_t M, int32_t N,
                                     int32_t dtype, void* stream) {
  if (N < 64 || N > 32768 || N % 64 != 0)
    return fail(VQ_ERR_INVALID_ARG, "N=%d must be a multiple of 64 in [64, 32768]", N);
  if (M < 0) return fail(VQ_ERR_INVALID_ARG, "M=%d is negative", M);
  if (dtype != VQ_F16 && dtype != VQ_BF16) return fail(VQ_ERR_INVALID_ARG, "dtype=%d", dtype);
  vq_status st;
  if ((st = check_ptr(y, "y")) || (st = check_ptr(y_out, "y_out")) || (st = check_ptr(signs, "signs"))) return st;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(y), b0 = reinterpret_cast<uintptr_t>(y_out);
  const uintptr_t bytes = (uintptr_t)M * N * 2;
  if (a0 != b0 && a0 < b0 + bytes && b0 < a0 + bytes)
    return fail(VQ_ERR_INVALID_ARG, "y_out partially overlaps y");
  if (M == 0) return VQ_OK;
  cudaError_t e = vq::launch_rht_output(y, y_out, signs, M, N, dtype, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "vq_rht_apply_output launch");
  return VQ_OK;
}

VQ_API vq_status vq_rht_apply_output_sharded(const void* y, void* y_out, const int8_t* signs, int32_t M, int32_t N,
                                             const int32_t* shard_n, int32_t nshards, int32_t dtype, void* stream) {
  if (shard_n == nullptr) return fail(VQ_ERR_INVALID_ARG, "shard_n is NULL");
  if (nshards < 1 || nshards > vq::kRhtMaxShards)
    return fail(VQ_ERR_INVALID_ARG, "nshards=%d outside [1, %d]", nshards, vq::kRhtMaxShards);
  vq::RhtShards sh{};
  sh.n = nshards;
  int64_t total = 0;
  for (int i = 0; i < nshards; ++i) {
    const int w = shard_n[i];
    if (w < 64 || w > 32768 || w % 64 != 0)
      return fail(VQ_ERR_INVALID_ARG, "shard_n[%d]=%d must be a multiple of 64 in [64, 32768]", i, w);
    sh.off[i] = (int)total;
    total += w;
  }
  if (total != N) return fail(VQ_ERR_INVALID_ARG, "the shards add up to %lld columns, N=%d", (long long)total, N);
  sh.off[nshards] = N;
  if (M < 0) return fail(VQ_ERR_INVALID_ARG, "M=%d is negative", M);
  if (dtype != VQ_F16 && dtype != VQ_BF16) return fail(VQ_ERR_INVALID_ARG, "dtype=%d", dtype);
  vq_status st;
  if ((st = check_ptr(y, "y")) || (st = check_ptr(y_out, "y_out")) || (st = check_ptr(signs, "signs"))) return st;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(y), b0 = reinterpret_cast<uintptr_t>(y_out);
  const uintptr_t bytes = (uintptr_t)M * N * 2;
  if (a0 != b0 && a0 < b0 + bytes && b0 < a0 + bytes) return fail(VQ_ERR_INVALID_ARG, "y_out partially overlaps y");
  if (M == 0) return VQ_OK;
  cudaError_t e = vq::launch_rht_output_shards(y, y_out, signs, M, N, sh, dtype, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "vq_rht_apply_output_sharded launch");
  return VQ_OK;
}

VQ_API vq_status vq_encode(const vq_linear_desc* desc, const float* w, const void* scales,
                           const vq_codebooks* codebooks, uint8_t* lo, uint8_t* hi4, uint8_t* s2, uint16_t* idx16,
                           void* stream) {
  if (desc == nullptr) return fail(VQ_ERR_INVALID_ARG, "desc is NULL");
  vq_linear_desc d = *desc;  // the fields a forward needs but the encoder does not use
  d.act_dtype = VQ_F16;
  d.max_M = 1;
  d.rht = 0;
  vq_status st;
  if ((st = validate_desc(&d))) return st;
  if (d.fmt == VQ_FMT_VQ16_RVQ) return fail(VQ_ERR_UNSUPPORTED, "the encoder takes the single-plane formats only");
  if ((st = check_ptr(w, "w")) || (st = validate_codebooks(d, codebooks, scales))) return st;
  if (d.fmt == VQ_FMT_VQ16) {
    if ((st = check_ptr(idx16, "idx16"))) return st;
  } else {
    if ((st = check_ptr(lo, "lo")) || (st = check_ptr(hi4, "hi4"))) return st;
    if (d.fmt == VQ_FMT_RVQ12_4 && (st = check_ptr(s2, "s2"))) return st;
  }
  vq::EncodeArgs a{};
  a.w = w;
  a.scales = static_cast<const uint16_t*>(scales);
  a.cb1 = static_cast<const uint16_t*>(codebooks->cb1);
  a.cb2 = d.fmt == VQ_FMT_RVQ12_4 ? static_cast<const uint16_t*>(codebooks->cb2) : nullptr;
  a.lo = lo;
  a.hi4 = hi4;
  a.s2 = s2;
  a.idx16 = idx16;
  a.N = d.N;
  a.K = d.K;
  a.fmt = d.fmt;
  a.scale_group = d.scale_group;
  cudaError_t e = vq::launch_encode(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "vq_encode launch");
  return VQ_OK;
}

VQ_API vq_status vq_linear_check(vq_linear_t h, void* stream) {
  if (h == nullptr) return fail(VQ_ERR_INVALID_ARG, "handle is NULL");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  uint32_t flag = 0;
  e = cudaMemcpy(&flag, h->err, sizeof flag, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the error word");
  if (flag) {
    // A forward that gave up may have left completion counters or the table
    // kernel's arrival counter part-way: clear them with the flag (one
    // allocation), so the handle is usable again.
    e = cudaMemset(h->err, 0, sizeof(uint32_t) * (2 + (size_t)h->num_tickets + (size_t)h->num_sync));
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "clearing the error word and the counters");
    return fail(VQ_ERR_TIMEOUT, "a bounded device wait gave up (flag 0x%x)", flag);
  }
  return VQ_OK;
}

VQ_API vq_status vq_debug_unpack(vq_linear_t h, const vq_planes* planes, uint16_t* i1_out, uint8_t* i2_out,
                                 void* stream) {
  if (h == nullptr) return fail(VQ_ERR_INVALID_ARG, "handle is NULL");
  vq_status st;
  if ((st = validate_planes(h->d, planes)) || (st = check_ptr(i1_out, "i1_out"))) return st;
  if ((st = check_device(h))) return st;
  vq::LayerArgs a = make_args(h->d, planes, nullptr, nullptr);
  cudaError_t e = vq::launch_debug_unpack(a, i1_out, i2_out, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "vq_debug_unpack launch");
  return VQ_OK;
}

VQ_API vq_status vq_debug_wait_timeout(vq_linear_t h, void* stream) {
  if (h == nullptr) return fail(VQ_ERR_INVALID_ARG, "handle is NULL");
  vq_status st;
  if ((st = check_device(h))) return st;
  cudaError_t e = vq::launch_debug_wait_timeout(h->err, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "vq_debug_wait_timeout launch");
  return VQ_OK;
}

VQ_API vq_status vq_debug_dequant(vq_linear_t h, const vq_planes* planes, const vq_codebooks* codebooks,
                                  const void* scales, void* w_out, int32_t wdt, void* stream) {
  if (h == nullptr) return fail(VQ_ERR_INVALID_ARG, "handle is NULL");
  if (wdt != VQ_F16 && wdt != VQ_BF16) return fail(VQ_ERR_INVALID_ARG, "wdt=%d", wdt);
  vq_status st;
  if ((st = validate_planes(h->d, planes)) || (st = validate_codebooks(h->d, codebooks, scales)) ||
      (st = check_ptr(w_out, "w_out")))
    return st;
  if ((st = check_device(h))) return st;
  vq::LayerArgs a = make_args(h->d, planes, codebooks, scales);
  cudaError_t e = vq::launch_debug_dequant(a, w_out, wdt, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "vq_debug_dequant launch");
  return VQ_OK;
}

// ---------------------------------------------------------------- no-allocation forward
//
// vq_linear_forward_noalloc runs the same warp-MMA GEMV kernel as
// vq_linear_forward (path VQ_PATH_GEMV) but takes its split-K scratch from a
// fixed buffer compiled into this library instead of from a handle, so a call
// never allocates device or host memory.
namespace {

constexpr size_t kNoAllocPartialBytes = size_t(4) << 20;  // split-K partial sums (fp32)
constexpr int kNoAllocTickets = 4096;                     // per-row-tile completion counters
constexpr int kNoAllocMaxDevices = 64;

// One copy per device (the module is loaded into each device's context).
// Partial sums first, then the tickets, which must be zero whenever no call is
// running: set-up clears them and every call leaves them zero.
static __device__ __align__(256) unsigned char
    g_noalloc_scratch[kNoAllocPartialBytes + kNoAllocTickets * sizeof(uint32_t)];

struct NoAllocDevice {
  bool ready;
  unsigned char* scratch;  // device address of g_noalloc_scratch on this device
  vq::DeviceInfo dev;
};
std::mutex g_noalloc_mu;
NoAllocDevice g_noalloc[kNoAllocMaxDevices];

// First use on a device (which must be current): look up the buffer's address,
// zero the tickets and wait for that to finish.  Later calls only read the cache.
vq_status noalloc_device(const NoAllocDevice** out) {
  int cur = -1;
  cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (cur < 0 || cur >= kNoAllocMaxDevices)
    return fail(VQ_ERR_UNSUPPORTED, "device %d: the no-allocation path supports devices 0..%d", cur,
                kNoAllocMaxDevices - 1);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocDevice& d = g_noalloc[cur];
  if (!d.ready) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, cur);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, cur);
    if (major != 10 || minor != 0)
      return fail(VQ_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a only", cur, major,
                  minor);
    vq::DeviceInfo info{};
    info.device = cur;
    cudaDeviceGetAttribute(&info.num_sms, cudaDevAttrMultiProcessorCount, cur);
    cudaDeviceGetAttribute(&info.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, cur);
    unsigned char* ptr = nullptr;
    e = cudaGetSymbolAddress((void**)&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-allocation scratch)");
    e = cudaMemset(ptr + kNoAllocPartialBytes, 0, kNoAllocTickets * sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "clearing the no-allocation tickets");
    d.scratch = ptr;
    d.dev = info;
    d.ready = true;
  }
  *out = &d;
  return VQ_OK;
}

}  // namespace

VQ_API vq_status vq_linear_forward_noalloc(const vq_linear_desc* desc, const void* x, const vq_planes* planes,
                                           const vq_codebooks* codebooks, const void* scales, void* y, int32_t M,
                                           void* stream) {
  vq_status st = validate_desc(desc);
  if (st == VQ_OK && desc->corr)
    return fail(VQ_ERR_UNSUPPORTED, "the sparse correction needs a handle's buffer: use vq_linear_forward");
  if (st) return st;
  const vq_linear_desc& d = *desc;
  if (M < 0 || M > 16) return fail(VQ_ERR_INVALID_ARG, "M=%d outside [0, 16] (the no-allocation path)", M);
  if ((st = check_ptr(x, "x")) || (st = check_ptr(y, "y")) || (st = validate_planes(d, planes)) ||
      (st = validate_codebooks(d, codebooks, scales)))
    return st;
  if (x == y) return fail(VQ_ERR_INVALID_ARG, "y must not alias x");
  if (M == 0) return VQ_OK;
  const NoAllocDevice* nd = nullptr;
  if ((st = noalloc_device(&nd))) return st;
  vq::Plan p{};
  if (!vq::plan_forward(d, nd->dev, M, VQ_PATH_GEMV, &p))
    return fail(VQ_ERR_UNSUPPORTED, "the GEMV path cannot run M=%d", M);
  if (p.scratch_bytes > kNoAllocPartialBytes || p.tickets > kNoAllocTickets)
    return fail(VQ_ERR_UNSUPPORTED,
                "N=%d, K=%d, M=%d needs %zu bytes of split-K scratch and %d tickets; the no-allocation buffer "
                "holds %zu bytes and %d tickets (use vq_linear_forward with a handle)",
                d.N, d.K, M, p.scratch_bytes, p.tickets, kNoAllocPartialBytes, kNoAllocTickets);
  vq::LayerArgs a = make_args(d, planes, codebooks, scales);
  a.x = x;
  a.y = y;
  a.M = M;
  cudaError_t e = vq::launch_gemv(a, p, reinterpret_cast<float*>(nd->scratch),
                                  reinterpret_cast<uint32_t*>(nd->scratch + kNoAllocPartialBytes),
                                  static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "vq_linear_forward_noalloc launch");
  return VQ_OK;
}
