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

// Split view of warp gw: {s0, s1, t_first, t_last, gf0, gl0, gf1, gl1}.
extern "C" void probe_warp_split(int gw, int S, int G, int KB, int* out) {
    q4::WarpSplit sp;
    sp.init(gw, q4::make_split(S, G), KB);
    const int v[8] = {sp.s0, sp.s1, sp.t_first, sp.t_last, sp.gf0, sp.gl0, sp.gf1, sp.gl1};
    for (int i = 0; i < 8; ++i) out[i] = v[i];
}
extern "C" int probe_cta_combiner(int gw, int e, int S, int G, int KB, int warps) {
    q4::WarpSplit sp;
    sp.init(gw, q4::make_split(S, G), KB);
    return q4::cta_combiner(sp, e, gw, gw / warps * warps) ? 1 : 0;
}
extern "C" int probe_park_slot_read(int gw, int w, int t, int S, int G, int KB) {
    q4::WarpSplit sp;
    sp.init(gw, q4::make_split(S, G), KB);
    return q4::park_slot_read(sp, gw, w, t);
}
extern "C" int probe_cta_slot_write(int c, int t, int KB, int S, int G, int warps) {
    return q4::cta_slot_write(c, t, KB, q4::make_split(S, G), warps);
}
extern "C" int probe_cta_slot_read(int c, int cf, int t, int KB, int S, int G, int warps) {
    return q4::cta_slot_read(c, cf, t, KB, q4::make_split(S, G), warps);
}
extern "C" int probe_shared_tile_of_boundary(int b, int KB, int S, int G, int warps) {
    return q4::shared_tile_of_boundary(b, KB, q4::make_split(S, G), warps);
}
