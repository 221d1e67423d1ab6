// ws_header.cuh -- the first 256 bytes of every workspace: the call's status
// word (0 = ok, else an flce_status_t a kernel recorded) and the count of
// non-ignored rows, N_valid, the divisor of the mean loss.
#pragma once

namespace flce {

struct WsHeader {
  int status;
  int pad;
  long long n_valid;
};

}  // namespace flce
