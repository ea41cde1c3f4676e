// Status strings and version of the C ABI declared in include/smcsd.h.
#include "smcsd.h"

extern "C" const char* sd_status_string(sd_status s) {
  switch (s) {
    case SD_OK: return "ok";
    case SD_ERR_INVALID_ARG: return "invalid argument";
    case SD_ERR_CUDA: return "CUDA launch or runtime error";
    case SD_ERR_UNSUPPORTED: return "unsupported size";
  }
  return "unknown status";
}

extern "C" int sd_version(void) { return 200; }
