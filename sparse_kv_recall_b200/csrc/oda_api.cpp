// Status names and version of the liboda C ABI.
#include "oda.h"

extern "C" const char* oda_status_string(int code) {
  switch (code) {
    case ODA_OK: return "ODA_OK";
    case ODA_ERR_INVALID_ARG: return "ODA_ERR_INVALID_ARG";
    case ODA_ERR_UNSUPPORTED_SHAPE: return "ODA_ERR_UNSUPPORTED_SHAPE";
    case ODA_ERR_WORKSPACE_TOO_SMALL: return "ODA_ERR_WORKSPACE_TOO_SMALL";
    case ODA_ERR_CUDA: return "ODA_ERR_CUDA";
    case ODA_ERR_NOT_IMPLEMENTED: return "ODA_ERR_NOT_IMPLEMENTED";
    case ODA_DEV_BAD_BLOCK: return "ODA_DEV_BAD_BLOCK";
    case ODA_DEV_BAD_LEN: return "ODA_DEV_BAD_LEN";
    case ODA_DEV_BAD_KEEP_LIST: return "ODA_DEV_BAD_KEEP_LIST";
    case ODA_DEV_TIMEOUT: return "ODA_DEV_TIMEOUT";
    default: return "ODA_UNKNOWN_STATUS";
  }
}

extern "C" int oda_version(void) { return 100; }
