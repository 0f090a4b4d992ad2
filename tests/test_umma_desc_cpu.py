"""The tensor-core descriptors the SSD kernels build (csrc/ssm_umma.cuh) against the definitions
in CUTLASS's CuTe headers (UMMA::SmemDescriptor, UMMA::make_instr_desc), on the host: a small
program is compiled with nvcc (host code only) and prints both encodings for every operand shape
the kernels use. No GPU is involved; skipped where nvcc or the CuTe headers are absent."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "selective_state_space_34_b200", "csrc")


def _cute_include():
    import importlib.util
    spec = importlib.util.find_spec("flashinfer")  # locates the package without importing it
    if spec is None or not spec.origin:
        return None
    d = os.path.join(os.path.dirname(spec.origin), "data", "cutlass", "include")
    return d if os.path.exists(os.path.join(d, "cute", "arch", "mma_sm100_desc.hpp")) else None


PROGRAM = r'''
#include <cstdio>
#include <cute/arch/mma_sm100_desc.hpp>
#include "ssm_umma.cuh"
using namespace cute;
template <int M, int N, int AMN, int BMN> int check_instr() {
  constexpr auto am = AMN ? UMMA::Major::MN : UMMA::Major::K;
  constexpr auto bm = BMN ? UMMA::Major::MN : UMMA::Major::K;
  const uint32_t ref = uint32_t(UMMA::make_instr_desc<bfloat16_t, bfloat16_t, float, M, N, am, bm>());
  const uint32_t mine = ssm::umma_instr_desc_bf16_f32(M, N, AMN, BMN);
  std::printf("instr M=%d N=%d a_mn=%d b_mn=%d ref=%08x mine=%08x\n", M, N, AMN, BMN, ref, mine);
  return ref == mine ? 0 : 1;
}
int check_smem(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  UMMA::SmemDescriptor d;
  d.start_address_ = uint16_t(addr >> 4);
  d.leading_byte_offset_ = uint16_t(lbo >> 4);
  d.stride_byte_offset_ = uint16_t(sbo >> 4);
  d.version_ = 1;
  d.base_offset_ = 0;
  d.lbo_mode_ = 0;
  d.layout_type_ = uint8_t(UMMA::LayoutType::SWIZZLE_NONE);
  const uint64_t ref = uint64_t(d), mine = ssm::umma_smem_desc_bits(addr, lbo, sbo);
  std::printf("smem addr=%u lbo=%u sbo=%u ref=%016llx mine=%016llx\n", addr, lbo, sbo,
              (unsigned long long)ref, (unsigned long long)mine);
  return ref == mine ? 0 : 1;
}
int main() {
  int bad = 0;
  bad += check_instr<128, 64, 1, 1>();
  bad += check_instr<128, 128, 1, 1>();
  bad += check_instr<128, 128, 0, 0>();
  bad += check_instr<128, 64, 0, 1>();
  bad += check_instr<128, 128, 0, 1>();
  const uint32_t addrs[4] = {0u, 1024u, 65536u + 4096u, 229376u - 4096u};
  const uint32_t lbos[3] = {1024u, 2048u, 128u};
  for (uint32_t a : addrs)
    for (uint32_t l : lbos) bad += check_smem(a, l, 128u);
  std::printf("mismatches %d\n", bad);
  return bad;
}
'''


def test_descriptors_match_cute():
    inc = _cute_include()
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if inc is None or not os.path.exists(nvcc):
        pytest.skip("nvcc or the CuTe headers are not available")
    d = tempfile.mkdtemp(prefix="umma_")
    try:
        src = os.path.join(d, "check.cu")
        open(src, "w").write(PROGRAM)
        exe = os.path.join(d, "check")
        subprocess.run([nvcc, "-std=c++17", "-I" + inc, "-I" + CSRC, "-o", exe, src], check=True,
                       capture_output=True, timeout=600)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
        assert r.returncode == 0, r.stdout
        assert "mismatches 0" in r.stdout
    finally:
        shutil.rmtree(d, ignore_errors=True)
