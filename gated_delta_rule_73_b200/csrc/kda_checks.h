// kda_checks.h -- the host-side argument rules shared by every entry point of the C ABI.
#pragma once
#include "../../include/kda.h"

namespace kda {
// opts: dtype, known and compatible flag bits, finite scale, events array (KDA_OK or a status)
int check_opts(const kda_opts &o);
// sizes: non-negative, dk and dv in {64, 128}, byte offsets that cannot overflow, B * H within
// the chunk kernels' grid (KDA_OK or a status)
int check_dims(long long B, long long T, long long H, int dk, int dv);
}  // namespace kda
