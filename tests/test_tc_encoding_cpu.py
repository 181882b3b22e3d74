"""The tcgen05 descriptors of the GEMM kernel against an independent encoder.

The instruction descriptor (kind::f16, f16 A and B, fp32 accumulator, both
operands K-major) and the shared-memory matrix descriptor (K-major, 128-byte
swizzle, 8-row groups 1024 bytes apart) are built by the kernel header's own
constexpr functions; CUTLASS's CuTe headers define the same bit fields
independently (cute/arch/mma_sm100_desc.hpp: UMMA::InstrDescriptor,
UMMA::make_instr_desc, UMMA::SmemDescriptor).  A host program compiled with
nvcc compares the two for every MMA width the kernel uses (N = 16..256) and
for several start addresses.  Skipped when no CuTe header tree is installed.
"""
import importlib.util
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "q4_quantized_decode_b200", "csrc", "gemm_tc.cuh")

PROGRAM = r"""
#include <cstdio>
#include <cute/arch/mma_sm100_desc.hpp>
#include <cute/numeric/numeric_types.hpp>
#include "gemm_tc.cuh"
int main() {
    int bad = 0;
    for (int n = 16; n <= 256; n += 16) {
        auto d = cute::UMMA::make_instr_desc<cute::half_t, cute::half_t, float, 128, 0,
                                             cute::UMMA::Major::K, cute::UMMA::Major::K>();
        d.n_dim_ = n >> 3;
        if (d.desc_ != q4::tc_idesc_f16(128, n)) { printf("idesc n=%d\n", n); ++bad; }
    }
    const unsigned addrs[] = {0u, 1024u, 1056u, 65632u, 232448u};
    for (unsigned a : addrs) {
        cute::UMMA::SmemDescriptor s;
        s.version_ = 1;
        s.lbo_mode_ = 0;
        s.base_offset_ = 0;
        s.layout_type_ = uint8_t(cute::UMMA::LayoutType::SWIZZLE_128B);
        s.start_address_ = (uint16_t)(a >> 4);
        s.leading_byte_offset_ = 1;
        s.stride_byte_offset_ = 1024 >> 4;
        if (s.desc_ != q4::tc_sdesc_sw128(a)) { printf("sdesc a=%u\n", a); ++bad; }
    }
    printf("mismatches %d\n", bad);
    return bad;
}
"""


def cute_include():
    for pkg, rel in (("flashinfer", ("data", "cutlass", "include")),
                     ("tilelang", ("3rdparty", "cutlass", "include"))):
        spec = importlib.util.find_spec(pkg)
        if spec is None or not spec.submodule_search_locations:
            continue
        for loc in spec.submodule_search_locations:
            inc = os.path.join(loc, *rel)
            if os.path.exists(os.path.join(inc, "cute", "arch", "mma_sm100_desc.hpp")):
                return inc
    return None


def test_descriptors_match_cute(tmp_path):
    inc = cute_include()
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if inc is None or not os.path.exists(nvcc):
        pytest.skip("CuTe headers or nvcc not available")
    src = tmp_path / "enc.cu"
    src.write_text(PROGRAM)
    exe = tmp_path / "enc"
    subprocess.check_call([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-I", inc, "-I", os.path.dirname(HEADER), "-o", str(exe), str(src)],
                          stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout
    assert "mismatches 0" in r.stdout
