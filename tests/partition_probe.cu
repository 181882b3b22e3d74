// Host-side harness exposing the GEMV kernel's work-partition helpers (the
// same inline functions the kernel uses) to the CPU tests.
#include "../q4_quantized_decode_b200/csrc/gemv_dp2a.cuh"

extern "C" int probe_seg_begin(int g, int S, int G) { return q4::seg_begin(g, q4::make_split(S, G)); }
extern "C" int probe_warp_of_seg(int s, int S, int G) { return q4::warp_of_seg(s, q4::make_split(S, G)); }
extern "C" int probe_walk(int g0, int steps, int S, int G) {
    q4::SegWalker w;
    w.init(g0, q4::make_split(S, G));
    for (int i = 0; i < steps; ++i) w.next();
    return w.sb;
}
extern "C" int probe_xperm_pos(int j) { return q4::xperm_pos(j); }
