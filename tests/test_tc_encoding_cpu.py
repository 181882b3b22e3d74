"""The tcgen05 descriptors of the GEMM kernel against an independent encoder.

The instruction descriptor (kind::f16, f16 A and B, fp32 accumulator, both
operands K-major) and the shared-memory matrix descriptor (K-major, 128-byte
swizzle, 8-row groups 1024 bytes apart) are built by the kernel header's own
constexpr functions; CUTLASS's CuTe headers define the same bit fields
independently (cute/arch/mma_sm100_desc.hpp: UMMA::InstrDescriptor,
UMMA::make_instr_desc, UMMA::SmemDescriptor).  A host program compiled with
nvcc compares the two for every MMA width the kernel uses (N = 16..256) and
for several start addresses.  Skipped when no CuTe header tree is installed.

The tcgen05 small-M kernel's B descriptor (K-major, no swizzle, 32-byte rows
in 8-row x 16-byte core matrices, the K-adjacent one 128 bytes on, the next
8-row group 256 bytes on) is checked against CuTe's own reading of such a
layout: UMMA::make_umma_desc<Major::K> (cute/atom/mma_traits_sm100.hpp)
derives the leading and stride offsets from a CuTe layout written with
exactly those strides, so a swap of the two offsets fails; its kind::i8
instruction descriptor (signed 8-bit A and B, int32 accumulator) against
UMMA::make_instr_desc<int8_t, int8_t, int32_t, ...>.  (On the host CuTe cannot read a shared-
memory address -- it prints an error and uses 0 -- so the start address is
compared at 0 there and field by field elsewhere.)
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
#include <cute/atom/mma_traits_sm100.hpp>
#include "gemm_tc.cuh"
#include "gemv_tcs.cuh"
int main() {
    using namespace cute;
    int bad = 0;
    {
        // The small-M kernel's B operand: rows of 32 signed bytes (K = 32);
        // row-in-group stride 16 bytes, 8-row group stride 256; K: 16
        // contiguous, the next chunk 128 bytes on.
        auto mma_layout = make_layout(make_shape(make_shape(Int<8>{}, Int<4>{}), make_shape(Int<16>{}, Int<2>{})),
                                      make_stride(make_stride(Int<16>{}, Int<256>{}), make_stride(Int<1>{}, Int<128>{})));
        auto e = UMMA::make_umma_desc<UMMA::Major::K>(
            make_tensor(make_smem_ptr(static_cast<int8_t*>(nullptr)), mma_layout));
        if (e.desc_ != q4::tcs_sdesc(0u)) { printf("tcs sdesc layout\n"); ++bad; }
        for (unsigned a : {0u, 128u, 1040u, 114688u, 229360u}) {
            UMMA::SmemDescriptor s = e;
            s.start_address_ = (uint16_t)(a >> 4);
            if (s.desc_ != q4::tcs_sdesc(a)) { printf("tcs sdesc a=%u\n", a); ++bad; }
        }
        for (int r = 0; r < 32; ++r)
            for (int k = 0; k < 2; ++k)
                if ((int)q4::tcs_core_off(r, k) != (int)mma_layout(make_coord(make_coord(r % 8, r / 8), make_coord(0, k)))) {
                    printf("tcs core offset r=%d k=%d\n", r, k);
                    ++bad;
                }
        for (int n = 16; n <= 32; n += 16) {
            auto d = cute::UMMA::make_instr_desc<int8_t, int8_t, int32_t, 128, 16,
                                                 cute::UMMA::Major::K, cute::UMMA::Major::K>();
            d.n_dim_ = n >> 3;
            if (d.desc_ != q4::tcs_idesc_i8(n)) { printf("tcs idesc n=%d\n", n); ++bad; }
        }
    }
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
