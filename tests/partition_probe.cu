// Host-side harness exposing the GEMV kernel's work-partition helpers (the
// same inline functions the kernel uses) to the CPU tests.
#include "../q4_quantized_decode_b200/csrc/gemv_dp2a.cuh"

extern "C" int probe_seg_begin(int g, int S, int G) { return q4::seg_begin(g, S, G); }
extern "C" int probe_warp_of_seg(int s, int S, int G) { return q4::warp_of_seg(s, S, G); }
extern "C" int probe_xperm_pos(int j) { return q4::xperm_pos(j); }
