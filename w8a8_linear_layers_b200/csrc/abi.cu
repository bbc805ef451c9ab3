// abi.cu -- library-wide entry points: status names, the thread-local error
// detail, the ABI version and the device check shared by every call.
#include "common.cuh"

#include <string.h>

namespace w8a8 {

static thread_local char g_detail[256] = "";

void set_detail(const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof g_detail, fmt, ap);
    va_end(ap);
}

sq_status check_device(int *sm_count) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(SQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    static int cache_major[64], cache_minor[64], cache_sms[64];
    static bool cached[64];
    int major, minor, sms;
    if (dev < 64 && cached[dev]) {
        major = cache_major[dev];
        minor = cache_minor[dev];
        sms = cache_sms[dev];
    } else {
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return fail(SQ_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
        if (dev < 64) {
            cache_major[dev] = major;
            cache_minor[dev] = minor;
            cache_sms[dev] = sms;
            cached[dev] = true;
        }
    }
    if (major != 10 || minor != 0)
        return fail(SQ_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a (B200)", dev,
                    major, minor);
    *sm_count = sms;
    return SQ_OK;
}

}  // namespace w8a8

extern "C" const char *sq_status_string(sq_status s) {
    switch (s) {
    case SQ_OK: return "SQ_OK";
    case SQ_ERR_NULL: return "SQ_ERR_NULL";
    case SQ_ERR_SHAPE: return "SQ_ERR_SHAPE";
    case SQ_ERR_DTYPE: return "SQ_ERR_DTYPE";
    case SQ_ERR_ALIGN: return "SQ_ERR_ALIGN";
    case SQ_ERR_ARG: return "SQ_ERR_ARG";
    case SQ_ERR_UNSUPPORTED: return "SQ_ERR_UNSUPPORTED";
    case SQ_ERR_CUDA: return "SQ_ERR_CUDA";
    case SQ_ERR_DEVICE: return "SQ_ERR_DEVICE";
    }
    return "SQ_ERR_UNKNOWN";
}

extern "C" const char *sq_last_error_detail(void) { return w8a8::g_detail; }

extern "C" int sq_abi_version(void) { return 1; }

extern "C" sq_status sq_debug_status(void *stream, uint64_t *nonfinite_out, uint64_t *index_out, int *enabled_out) {
    if (!nonfinite_out || !index_out || !enabled_out) return w8a8::fail(SQ_ERR_NULL, "sq_debug_status: NULL pointer");
#ifdef W8A8_DEBUG
    int sms;
    sq_status st = w8a8::check_device(&sms);
    if (st != SQ_OK) return st;
    cudaStream_t cs = (cudaStream_t)stream;
    unsigned long long total[2] = {0ull, 0ull};
    cudaError_t (*readers[])(cudaStream_t, unsigned long long (&)[2]) = {
        w8a8::dbg_take_smooth, w8a8::dbg_take_quant_act, w8a8::dbg_take_ssz, w8a8::dbg_take_ssz_asym};
    for (auto rd : readers) {
        unsigned long long c[2];
        const cudaError_t e = rd(cs, c);
        if (e != cudaSuccess) return w8a8::fail(SQ_ERR_CUDA, "sq_debug_status: %s", cudaGetErrorString(e));
        total[0] += c[0];
        total[1] += c[1];
    }
    *nonfinite_out = total[0];
    *index_out = total[1];
    *enabled_out = 1;
#else
    (void)stream;
    *nonfinite_out = 0;
    *index_out = 0;
    *enabled_out = 0;
#endif
    return SQ_OK;
}
