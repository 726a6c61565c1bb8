// Library-wide host plumbing: error strings, device checks, batch grouping,
// workspace carving, default parameters.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <utility>

#include "internal.h"
#include "umma.cuh"

namespace ouo {

static thread_local char g_last_error[1024] = "";

int set_error(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return code;
}

void clear_error() { g_last_error[0] = 0; }

static std::atomic<unsigned long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int num_sms() {
  static std::atomic<int> cached[64];  // zero-initialized (static storage)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64) {
    const int c = cached[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
      cudaSuccess)
    n = 148;
  if (dev >= 0 && dev < 64) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

int require_sm100() {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return set_error(OUO_ERR_NO_DEVICE, "no CUDA device: %s",
                     cudaGetErrorString(e));
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    return set_error(OUO_ERR_NO_DEVICE,
                     "device %d is sm_%d%d; this library is built for sm_100a",
                     dev, major, minor);
  return OUO_OK;
}

std::vector<Group> group_by_shape(const ouo_mat* mats, int nmat) {
  std::vector<Group> out;
  std::map<std::pair<int64_t, int64_t>, int> where;
  for (int i = 0; i < nmat; ++i) {
    auto key = std::make_pair(mats[i].rows, mats[i].cols);
    auto it = where.find(key);
    if (it == where.end()) {
      where[key] = (int)out.size();
      Group g;
      g.rows = mats[i].rows;
      g.cols = mats[i].cols;
      g.members.push_back(i);
      out.push_back(g);
    } else {
      out[it->second].members.push_back(i);
    }
  }
  return out;
}

int validate_dtype(int dtype, const char* name) {
  if (dtype != OUO_F32 && dtype != OUO_BF16)
    return set_error(OUO_ERR_INVALID_ARG, "%s: unknown dtype %d", name, dtype);
  return OUO_OK;
}

int validate_mats(const ouo_mat* mats, int nmat, int dtype, const char* name) {
  if (!mats)
    return set_error(OUO_ERR_INVALID_ARG, "%s: NULL batch array", name);
  OUO_TRY(validate_dtype(dtype, name));
  size_t es = elem_size(dtype);
  for (int i = 0; i < nmat; ++i) {
    const ouo_mat& m = mats[i];
    if (!m.ptr)
      return set_error(OUO_ERR_INVALID_ARG, "%s[%d]: NULL pointer", name, i);
    if (m.rows < 1 || m.cols < 1)
      return set_error(OUO_ERR_INVALID_ARG, "%s[%d]: empty shape %lld x %lld",
                       name, i, (long long)m.rows, (long long)m.cols);
    if (m.rows > (int64_t)1 << 31 || m.cols > (int64_t)1 << 31)
      return set_error(OUO_ERR_INVALID_ARG, "%s[%d]: shape too large", name, i);
    if (m.ld < m.cols)
      return set_error(OUO_ERR_INVALID_ARG, "%s[%d]: ld %lld < cols %lld",
                       name, i, (long long)m.ld, (long long)m.cols);
    if (((uintptr_t)m.ptr) % es != 0)
      return set_error(OUO_ERR_INVALID_ARG,
                       "%s[%d]: pointer not aligned to its element size", name,
                       i);
  }
  return OUO_OK;
}

bool vec16(const ouo_mat& m, int dtype) {
  return ((uintptr_t)m.ptr) % 16 == 0 && ((size_t)m.ld * elem_size(dtype)) % 16 == 0;
}

int validate_same_shapes(const ouo_mat* a, const ouo_mat* b, int nmat,
                         const char* na, const char* nb) {
  for (int i = 0; i < nmat; ++i)
    if (a[i].rows != b[i].rows || a[i].cols != b[i].cols)
      return set_error(OUO_ERR_INVALID_ARG,
                       "%s[%d] is %lld x %lld but %s[%d] is %lld x %lld", na,
                       i, (long long)a[i].rows, (long long)a[i].cols, nb, i,
                       (long long)b[i].rows, (long long)b[i].cols);
  return OUO_OK;
}

Buf Arena::take(int dtype, int64_t nb, int64_t rows, int64_t cols) {
  Buf b;
  b.dtype = dtype;
  b.nb = nb;
  b.rows = rows;
  b.cols = cols;
  // rows padded to 16 bytes (TMA stride rule), matrices to 256 bytes
  int64_t per16 = 16 / (int64_t)elem_size(dtype);
  b.ld = ceil_div(cols, per16) * per16;
  int64_t per256 = 256 / (int64_t)elem_size(dtype);
  b.stride = ceil_div(rows * b.ld, per256) * per256;
  size_t bytes = (size_t)nb * (size_t)b.stride * elem_size(dtype);
  used = align_up(used, 256);
  b.p = measuring ? nullptr : base + used;
  used += bytes;
  return b;
}

namespace {

// Waits on an mbarrier that nothing arrives on, bounded by limit_ns, then
// reports OUO_STATUS_TIMEOUT: the same bounded wait the GEMM pipeline uses,
// made to run out on purpose.
__global__ void wait_timeout_kernel(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    ptx::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !ptx::mbar_wait_timed(&bar, 0, limit_ns))
    report_status(status, OUO_STATUS_TIMEOUT);
}

}  // namespace
}  // namespace ouo

extern "C" {

int ouo_debug_wait_timeout(int* dev_status, unsigned long long limit_ns,
                           void* stream) {
  ouo::clear_error();
  if (!dev_status)
    return ouo::set_error(OUO_ERR_INVALID_ARG, "dev_status is required");
  if (limit_ns > 1000000000ull)
    return ouo::set_error(OUO_ERR_INVALID_ARG, "limit above 1 s");
  OUO_TRY(ouo::require_sm100());
  ouo::wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(dev_status, limit_ns);
  OUO_CHECK_LAUNCH();
  return OUO_OK;
}

int ouo_version(void) { return OUO_VERSION; }

const char* ouo_last_error(void) { return ouo::g_last_error; }

int ouo_timing_enable(int on) {
  ouo::clear_error();
  return ouo::gemm_timing_enable(on);
}

int ouo_timing_read(int kind, int* launches, double* total_ms, double* flops) {
  ouo::clear_error();
  return ouo::gemm_timing_read(kind, launches, total_ms, flops);
}

unsigned long long ouo_launch_count(void) {
  return ouo::g_launches.load(std::memory_order_relaxed);
}

void ouo_ns_default(ouo_ns_params* p) {
  if (!p) return;
  std::memset(p, 0, sizeof(*p));
  p->a = 3.4445f;
  p->b = -4.7750f;
  p->c = 2.0315f;
  p->iters = 5;
  p->safety = 1.0f;
  p->eps = 1e-7f;
  p->normalize = 1;
  p->precision = OUO_PREC_BF16;
  p->n_restart = 1;
  p->restart_after[0] = 3;
}

void ouo_dion_default(ouo_dion_params* p) {
  if (!p) return;
  std::memset(p, 0, sizeof(*p));
  p->rank = 256;
  p->mu = 0.95f;
  p->beta = 1.0f;
  p->lr = 0.01f;
  p->wd = 0.0f;
  p->norm_mode = OUO_DION_COLNORM;
  p->eps = 1e-8f;
}

int64_t dion3_num_selected(int64_t rows, double rho) {
  if (rows < 1 || !(rho > 0.0) || rho > 1.0) return -1;
  double x = rho * (double)rows - 1e-9;
  int64_t k = (int64_t)x;
  if ((double)k < x) k += 1;  // ceil
  if (k < 1) k = 1;
  if (k > rows) k = rows;
  return k;
}

}  // extern "C"
