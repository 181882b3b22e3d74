"""Host checks of the GEMV kernel's work partition (compiled from the
kernel's own header, run on the CPU): every segment has exactly one owning
warp, the tile contributor ranges contain only owning warps, and the arrival
bookkeeping (slots, counts) is consistent."""
import ctypes
import os
import subprocess

import pytest

from q4_quantized_decode_b200 import build_ext

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    out = tmp_path_factory.mktemp("probe") / "libprobe.so"
    subprocess.check_call([build_ext.nvcc(), "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
                           "-gencode", "arch=compute_100a,code=sm_100a",
                           os.path.join(HERE, "partition_probe.cu"), "-o", str(out)])
    lib = ctypes.CDLL(str(out))
    for f in ("probe_seg_begin", "probe_warp_of_seg"):
        getattr(lib, f).argtypes = [ctypes.c_int] * 3
    lib.probe_walk.argtypes = [ctypes.c_int] * 4
    lib.probe_warp_split.argtypes = [ctypes.c_int] * 4 + [ctypes.POINTER(ctypes.c_int)]
    lib.probe_cta_combiner.argtypes = [ctypes.c_int] * 6
    lib.probe_park_slot_read.argtypes = [ctypes.c_int] * 6
    lib.probe_cta_slot_write.argtypes = [ctypes.c_int] * 6
    lib.probe_cta_slot_read.argtypes = [ctypes.c_int] * 7
    lib.probe_shared_tile_of_boundary.argtypes = [ctypes.c_int] * 5
    lib.probe_xperm_pos.argtypes = [ctypes.c_int]
    return lib


CASES = [(1, 1), (4, 4), (4, 2), (17, 5), (1024, 256), (25600, 2368), (87040, 2368),
         (174080, 2368), (160, 148), (1088 * 160, 2368), (7, 7), (100, 99)]


@pytest.mark.parametrize("S,G", CASES)
def test_partition_is_exact_cover(probe, S, G):
    begins = [probe.probe_seg_begin(g, S, G) for g in range(G + 1)]
    assert begins[0] == 0 and begins[G] == S
    for g in range(G):
        assert begins[g + 1] - begins[g] >= 1          # G <= S: no empty warp
    for s in range(0, S, max(1, S // 5000)):
        g = probe.probe_warp_of_seg(s, S, G)
        assert begins[g] <= s < begins[g + 1]


@pytest.mark.parametrize("S,G,KB", [(4, 4, 2), (25600, 2368, 160), (87040, 2368, 544),
                                    (174080, 2368, 160), (1024, 256, 32), (8192, 2048, 1),
                                    (12, 12, 3), (99, 50, 9)])
def test_arrival_bookkeeping(probe, S, G, KB):
    begins = [probe.probe_seg_begin(g, S, G) for g in range(G + 1)]
    T = S // KB
    arrivals = [0] * T
    slots_used = set()
    for g in range(G):
        s0, s1 = begins[g], begins[g + 1]
        t_first, t_last = s0 // KB, (s1 - 1) // KB
        for t in range(t_first, t_last + 1):
            gf = probe.probe_warp_of_seg(t * KB, S, G)
            gl = probe.probe_warp_of_seg(t * KB + KB - 1, S, G)
            whole = gf == gl
            if t not in (t_first, t_last):
                assert whole                        # middle tiles are owned whole
            if not whole:
                slot = 0 if t == t_first else 1
                assert (g, slot) not in slots_used
                slots_used.add((g, slot))
                arrivals[t] += 1
    for t in range(T):
        gf = probe.probe_warp_of_seg(t * KB, S, G)
        gl = probe.probe_warp_of_seg(t * KB + KB - 1, S, G)
        assert arrivals[t] == (0 if gf == gl else gl - gf + 1)
        for gg in range(gf, gl + 1):                # the reducer's slot choice
            if gf != gl:
                sl = 0 if begins[gg] // KB == t else 1
                assert (gg, sl) in slots_used


BIG = [(2**31 - 1, 2368), (2**31 - 1, 65535), (123456789, 40000), (2**30 + 7, 3),
       (5 * 2**20 + 3, 65535), (2**24, 2**16 - 1), (65535, 65535), (2, 2), (3, 2)]


@pytest.mark.parametrize("S,G", BIG)
def test_reciprocal_division_is_exact(probe, S, G):
    """seg_begin / warp_of_seg divide by multiplying with a 64-bit reciprocal;
    check them against exact integer division, including splits whose
    numerators need 64 bits."""
    import random
    rng = random.Random(S * 7919 + G)
    gs = [0, 1, G - 1, G] + [rng.randrange(G + 1) for _ in range(300)]
    for g in gs:
        assert probe.probe_seg_begin(g, S, G) == g * S // G
    ss = [0, 1, S - 1, S - 2 if S > 1 else 0] + [rng.randrange(S) for _ in range(300)]
    for s in ss:
        assert probe.probe_warp_of_seg(s, S, G) == ((s + 1) * G - 1) // S


@pytest.mark.parametrize("S,G", [(25600, 2368), (87040, 2368), (17, 5), (100, 99), (9, 1)])
def test_walker_matches_seg_begin(probe, S, G):
    for g0 in (0, 1, G // 3, G - 1):
        for steps in range(0, min(G - g0, 40) + 1):
            assert probe.probe_walk(g0, steps, S, G) == (g0 + steps) * S // G


def test_xperm_is_a_permutation_grouping_lane_words(probe):
    pos = [probe.probe_xperm_pos(j) for j in range(32)]
    assert sorted(pos) == list(range(32))
    for c in range(4):
        group = {pos[j] for j in list(range(4 * c, 4 * c + 4)) + list(range(16 + 4 * c, 20 + 4 * c))}
        assert group == set(range(8 * c, 8 * c + 8))


def _split(probe, gw, S, G, KB):
    out = (ctypes.c_int * 8)()
    probe.probe_warp_split(gw, S, G, KB, out)
    return list(out)


@pytest.mark.parametrize("S,G,KB", [(25600, 2368, 160), (35840, 2368, 160), (174080, 2368, 160),
                                    (87040, 2368, 544), (12, 12, 3), (99, 50, 9), (994, 37, 7), (1001, 40, 7), (7 * 130, 148 * 16 // 3, 7),
                                    (5000, 333, 1), (160, 160, 160), (64, 64, 64), (165, 165, 5),
                                    (4096, 2368, 4096), (300, 150, 30), (2368 * 3, 2368, 2)])
def test_two_level_combine_bookkeeping(probe, S, G, KB):
    """Simulates the two-level combine of the M <= 2 kernel and of the
    persistent step with the kernel's own decision functions: every parked
    partial that is read was parked for that tile, every split tile is
    combined once per contributing CTA, CTA partial slots never collide and
    the reader finds them, and each tile shared by CTAs has exactly one
    writer of its output in a traced step."""
    W = 16
    T = S // KB
    sp = {gw: _split(probe, gw, S, G, KB) for gw in range(G)}
    parked = {}
    for gw, (s0, s1, tf, tl, gf0, gl0, gf1, gl1) in sp.items():
        assert s1 > s0
        for t, gf, gl in ((tf, gf0, gl0), (tl, gf1, gl1)):
            if gf != gl:
                parked[(gw, 0 if t == tf else 1)] = t
    combined, y_written, cta_parked = {}, [0] * T, {}
    for gw, (s0, s1, tf, tl, gf0, gl0, gf1, gl1) in sp.items():
        b, cta_lo = gw // W, gw // W * W
        for e, (t, gf, gl) in enumerate(((tf, gf0, gl0), (tl, gf1, gl1))):
            if not probe.probe_cta_combiner(gw, e, S, G, KB, W):
                continue
            assert gw == max(gf, cta_lo)                 # the CTA's first contributor
            w_to = min(gl, cta_lo + W - 1)
            for w in range(gw, w_to + 1):
                sl = probe.probe_park_slot_read(gw, w, t, S, G, KB)
                assert parked.get((w, sl)) == t
            assert (b, t) not in combined
            combined[(b, t)] = 1
            if gf >= cta_lo and gl <= cta_lo + W - 1:
                y_written[t] += 1
            else:
                slc = probe.probe_cta_slot_write(b, t, KB, S, G, W)
                assert (b, slc) not in cta_parked
                cta_parked[(b, slc)] = t
    for t in range(T):
        gf = probe.probe_warp_of_seg(t * KB, S, G)
        gl = probe.probe_warp_of_seg(t * KB + KB - 1, S, G)
        if gf == gl:
            assert y_written[t] == 0                      # written by its warp's flush
            continue
        cf, cl = gf // W, gl // W
        for c in range(cf, cl + 1):
            assert combined.get((c, t)) == 1
        if cf == cl:
            assert y_written[t] == 1
            continue
        assert y_written[t] == 0
        for c in range(cf, cl + 1):
            sl = probe.probe_cta_slot_read(c, cf, t, KB, S, G, W)
            assert cta_parked.get((c, sl)) == t
    # The persistent step's readers enumerate the shared tiles by CTA
    # boundary: each shared tile exactly once, named with its first CTA b-1.
    nb = (G + W - 1) // W
    named = {}
    for b in range(1, nb):
        t = probe.probe_shared_tile_of_boundary(b, KB, S, G, W)
        if t >= 0:
            assert t not in named
            named[t] = b
    shared = {t for t in range(T)
              if probe.probe_warp_of_seg(t * KB, S, G) // W != probe.probe_warp_of_seg(t * KB + KB - 1, S, G) // W}
    assert set(named) == shared
    for t, b in named.items():
        assert probe.probe_warp_of_seg(t * KB, S, G) // W == b - 1
