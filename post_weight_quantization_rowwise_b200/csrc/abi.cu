// abi.cu -- status strings, last CUDA error and version of the C ABI (iqq.h).
#include "common.cuh"

namespace iqq {
namespace {
thread_local int g_last_cuda_error = 0;
}
void set_last_cuda_error(cudaError_t e) { g_last_cuda_error = static_cast<int>(e); }
}  // namespace iqq

extern "C" const char* iqq_status_string(iqq_status status)
{
    switch (status) {
    case IQQ_OK: return "ok";
    case IQQ_ERR_NULL: return "a required pointer is NULL";
    case IQQ_ERR_SHAPE: return "invalid shape (negative, not a multiple of the block, or too large)";
    case IQQ_ERR_ALIGN: return "a pointer is not aligned as required";
    case IQQ_ERR_CUDA: return "CUDA launch failed (see iqq_last_cuda_error)";
    case IQQ_ERR_ARG: return "an argument is out of range";
    }
    return "unknown status";
}

extern "C" int iqq_last_cuda_error(void) { return iqq::g_last_cuda_error; }

extern "C" const char* iqq_version(void)
{
    return "iqq 0.1 sm_100a (built " __DATE__ " " __TIME__ ")";
}
