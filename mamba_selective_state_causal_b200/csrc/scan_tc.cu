// scan_tc.cu -- tensor-core (tcgen05/TMEM/TMA) path of the chunked scan.
#include "ssd_common.cuh"

namespace ssd {

bool tc_scan_supported(const ScanParams &, int) { return false; }

int launch_scan_tc(const ScanParams &, cudaStream_t) { return 6; }

}  // namespace ssd
