// sf_api.cu -- library-wide entry points of the C ABI (version, status strings).
#include "sf_host.h"

extern "C" const char *sf_status_string(int code)
{
    switch (code) {
    case SF_OK: return "ok";
    case SF_ERR_ARG: return "invalid argument (null pointer, size or shape)";
    case SF_ERR_ALIGN: return "misaligned pointer or leading dimension (16-byte rule)";
    case SF_ERR_UNSUPPORTED: return "size beyond what this build supports";
    case SF_ERR_CUDA: return "CUDA runtime error or failed launch";
    case SF_ERR_NO_DEVICE: return "no usable CUDA device is current";
    default: return "unknown status";
    }
}

extern "C" int sf_version(void) { return 10000; }
