// Status strings, device-status check and per-device SM count.
#include <mutex>

#include "common.cuh"

namespace st {

// SM budget of the launches this host thread issues (0: the whole device).
thread_local int t_sm_budget = 0;

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  int n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) {
    if (cache[dev] == 0) {
      int a = 0;
      if (cudaDeviceGetAttribute(&a, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || a <= 0) a = 148;
      cache[dev] = a;
    }
    n = cache[dev];
  }
  return t_sm_budget > 0 && t_sm_budget < n ? t_sm_budget : n;
}

}  // namespace st

ST_API st_status st_set_sm_budget(int sms) {
  if (sms < 0) return ST_ERR_SHAPE;
  st::t_sm_budget = sms;
  return ST_OK;
}

ST_API int st_get_sm_budget(void) { return st::t_sm_budget; }

ST_API const char *st_status_string(st_status s) {
  switch (s) {
    case ST_OK: return "ST_OK";
    case ST_ERR_NULL: return "ST_ERR_NULL: a required pointer is NULL";
    case ST_ERR_SHAPE: return "ST_ERR_SHAPE: a size is out of range or inconsistent";
    case ST_ERR_DIVISIBILITY: return "ST_ERR_DIVISIBILITY: P, N_T, N_S or H does not divide";
    case ST_ERR_DTYPE: return "ST_ERR_DTYPE: dtype or element size not supported";
    case ST_ERR_ALIGN: return "ST_ERR_ALIGN: pointer or pitch not aligned";
    case ST_ERR_UNSUPPORTED: return "ST_ERR_UNSUPPORTED: no kernel for this request";
    case ST_ERR_CUDA: return "ST_ERR_CUDA: the CUDA runtime reported an error";
    case ST_ERR_TIMEOUT: return "ST_ERR_TIMEOUT: a bounded device wait ran out";
  }
  return "unknown st_status";
}

ST_API int st_abi_version(void) { return 1; }

ST_API st_status st_check_device_status(st_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return ST_ERR_CUDA;
  cudaError_t err = cudaSuccess;
  unsigned int word = st::read_and_clear_attn_error(s, &err);
  if (err != cudaSuccess) return ST_ERR_CUDA;
  word |= st::read_and_clear_relayout_error(s, &err);
  if (err != cudaSuccess) return ST_ERR_CUDA;
  word |= st::read_and_clear_vmajor_error(s, &err);
  if (err != cudaSuccess) return ST_ERR_CUDA;
  return word ? ST_ERR_TIMEOUT : ST_OK;
}
