// scan_chunked.cu -- chunked (C = 64) tensor-core Gated DeltaNet scan.
#include "tr_internal.h"

namespace tr {

bool scan_chunked_supported(const ScanLaunch &p) {
  (void)p;
  return false;
}

cudaError_t launch_scan_chunked(const ScanLaunch &p, cudaStream_t s, std::string *err) {
  (void)p;
  (void)s;
  if (err) *err = "chunked scan not available";
  return cudaErrorNotSupported;
}

}  // namespace tr
