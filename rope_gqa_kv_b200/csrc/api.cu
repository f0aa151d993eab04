// api.cu -- status strings and version of the libgqa C ABI.
#include "common.cuh"

extern "C" const char *gqa_status_string(gqa_status s) {
    switch (s) {
        case GQA_OK: return "ok";
        case GQA_ERR_INVALID_ARG: return "invalid argument (null, size, alignment or Hq % Hkv)";
        case GQA_ERR_UNSUPPORTED: return "unsupported (head_dim must be 64, 96 or 128; sm_100 GPU)";
        case GQA_ERR_CAPACITY: return "positions or lengths exceed the cache capacity Lmax";
        case GQA_ERR_TIMEOUT: return "a bounded wait timed out";
        case GQA_ERR_CUDA: return "CUDA runtime or driver error";
        case GQA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    }
    return "unknown status";
}

extern "C" int gqa_version(void) { return 200; }
