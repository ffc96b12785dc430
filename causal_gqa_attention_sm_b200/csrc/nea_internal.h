// Library-internal interface between the attention entry points
// (nea_attn.cu) and the decoder-block steps (nea_block.cu): the per-device
// status word that nea_device_status() reads, the SM count, and the calling
// thread's device-side wait limit.
#pragma once

namespace nea_internal {

// Sets up (on first use) and returns the current device's status word and SM
// count; returns an NEA_* status.
int device_status_word(int** err, int* n_sm);
// The calling thread's limit for bounded device-side waits, nanoseconds.
long long wait_limit_ns();

}  // namespace nea_internal
