"""The C-ABI library builds for sm_100a, loads without a GPU, exports every declared symbol,
and rejects bad arguments on the host (no kernel is launched by these calls)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _build_module():
    import importlib.util

    spec = importlib.util.spec_from_file_location("pa_build", os.path.join(ROOT, "paged_kv_cache_475_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


B = _build_module()


@pytest.fixture(scope="module")
def lib():
    path = B.build()
    return ctypes.CDLL(path)


def declared_symbols():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"PA_API\s+[\w\s\*]+?\b(pa_\w+)\s*\(", text)
    return names


def test_header_declares_entry_points():
    names = set(declared_symbols())
    for n in ("pa_reshape_and_cache", "pa_decode", "pa_decode_splitkv", "pa_merge", "pa_prefill_chunk",
              "pa_slot_mapping", "pa_read_error_flags", "pa_status_string"):
        assert n in names


def test_exports_every_declared_symbol(lib):
    missing = [n for n in declared_symbols() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings_and_version(lib):
    lib.pa_status_string.restype = ctypes.c_char_p
    assert lib.pa_status_string(0) == b"PA_OK"
    for code in range(-7, 0):
        assert lib.pa_status_string(code).startswith(b"PA_ERR")
    assert lib.pa_version() >= 100


def test_num_partitions(lib):
    f = lib.pa_splitkv_num_partitions
    assert f(100000, 512) == 196
    assert f(512, 512) == 1
    assert f(513, 512) == 2
    assert f(0, 512) == 1
    assert f(10, 0) == 0


def test_splitkv_workspace_bytes(lib):
    """The section 8(b) workspace query: three fp32 parts, each rounded up to 256 bytes; 0 when invalid."""
    f = lib.pa_splitkv_workspace_bytes
    f.restype = ctypes.c_size_t
    r256 = lambda n: (n + 255) // 256 * 256  # noqa: E731
    # 100k split-KV shape: 4 x 32 rows, 196 partitions of 512 tokens, D = 128
    cells = 4 * 32 * 196
    assert f(4, 32, 128, 100000, 512) == r256(cells * 128 * 4) + 2 * r256(cells * 4)
    # one partition per row even for an empty context; a 1-cell part still takes 256 bytes
    assert f(1, 1, 64, 0, 512) == r256(64 * 4) + 2 * 256
    assert f(3, 5, 64, 513, 512) == r256(3 * 5 * 2 * 64 * 4) + 2 * r256(3 * 5 * 2 * 4)
    assert f(0, 32, 128, 4096, 512) == 0
    for bad in [(-1, 32, 128, 4096, 512), (4, 0, 128, 4096, 512), (4, 32, 0, 4096, 512), (4, 32, 128, -5, 512),
                (4, 32, 128, 4096, 0)]:
        assert f(*bad) == 0, bad
    # sizes that do not fit in size_t report 0 rather than a wrapped value
    assert f(2**31 - 1, 2**31 - 1, 2**31 - 1, 2**31 - 1, 16) == 0


def _noalloc_args(**kw):
    fake = ctypes.c_void_p(256)  # never dereferenced: every case below is refused on the host
    a = dict(out=fake, q=fake, k=fake, v=fake, bt=fake, mb=4, lens=fake, N=2, Hq=8, Hkv=2, D=128, B=16, P=10,
             part=512, np=4, scale=ctypes.c_float(0.1), dt=1, stream=None)
    a.update(kw)
    return list(a.values())


@pytest.mark.parametrize("kw,code", [
    # rows * partitions * (D + 2) * 4 bytes far beyond the 16 MiB array
    (dict(np=100_000), -5),
    # a product that would wrap 64 bits if formed naively: 65535 x 2^31-1 rows ...
    (dict(N=65535, Hq=2**31 - 1, Hkv=2**31 - 1, np=2**30), -5),
    (dict(N=65535, Hq=2**31 - 1, Hkv=2**31 - 1, np=2**30 + 1), -2),  # ... or a partition count past 2^30
    (dict(N=1, Hq=8, np=2**30 + 1), -2),
    (dict(N=65536), -2),
    (dict(part=24), -5), (dict(np=0), -5), (dict(out=None), -1),
])
def test_noalloc_rejects_oversized_or_absurd_shapes_on_host(lib, kw, code):
    """pa_decode_splitkv_noalloc refuses before any CUDA call (these run without a GPU)."""
    assert lib.pa_decode_splitkv_noalloc(*_noalloc_args(**kw)) == code


def _decode_args(**kw):
    fake = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    a = dict(out=fake, q=fake, k=fake, v=fake, bt=fake, mb=4, lens=fake, N=2, Hq=8, Hkv=2, D=128, B=16, P=10,
             scale=ctypes.c_float(0.1), dt=1, stream=None)
    a.update(kw)
    return list(a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(D=96), -4), (dict(B=24), -4), (dict(Hq=6, Hkv=4), -2), (dict(Hq=48, Hkv=2), -4),
    (dict(dt=7), -3), (dict(q=None), -1), (dict(N=-1), -2), (dict(q=ctypes.c_void_p(24)), -7),
])
def test_decode_rejects_bad_args_on_host(lib, kw, code):
    assert lib.pa_decode(*_decode_args(**kw)) == code


@pytest.mark.parametrize("cycles", [0, 999, 4_000_000_001, -5])
def test_starved_wait_selftest_rejects_wait_limits_out_of_range_on_host(lib, cycles):
    """The wait-limit self-test accepts 1000 .. 4e9 cycles and refuses the rest before any CUDA call."""
    fn = lib.pa_decode_selftest_starved_wait
    fn.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int, ctypes.c_void_p] + [ctypes.c_int] * 6 + [
        ctypes.c_float, ctypes.c_int, ctypes.c_longlong, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    a = _decode_args()
    assert fn(*a[:-1], cycles, None) == -2


def test_splitkv_rejects_bad_partition(lib):
    fake = ctypes.c_void_p(16)
    args = [fake, fake, fake, fake, fake, fake, fake, 4, fake, 2, 8, 2, 128, 16, 10, 24, 3,
            ctypes.c_float(0.1), 1, None]
    assert lib.pa_decode_splitkv(*args) == -5  # partition not a multiple of 16
    args[15] = 512
    args[16] = 0
    assert lib.pa_decode_splitkv(*args) == -5  # no partitions


def test_prefill_rejects_f32(lib):
    fake = ctypes.c_void_p(16)
    args = [fake, fake, fake, fake, fake, 4, fake, 2, 8, 8, 2, 128, 16, 10, ctypes.c_float(0.1), 0, None]
    assert lib.pa_prefill_chunk(*args) == -3


def test_zero_sized_calls_are_noops(lib):
    assert lib.pa_slot_mapping(None, None, 0, None, None, 0, 0, 16, None) == 0
    assert lib.pa_reshape_and_cache(None, None, None, None, None, 0, 10, 8, 128, 16, 1, None) == 0


def _sp_args(**kw):
    fake = ctypes.c_void_p(16)
    a = dict(out=fake, q=fake, k_new=None, v_new=None, kc=fake, vc=fake, bt=fake, mb=4, lens=fake, N=4, Hq=8,
             Hkv=2, D=128, B=16, P=10, prefix=64, group=2, po=fake, pm=fake, pl=fake, np=5,
             scale=ctypes.c_float(0.1), dt=1, stream=None)
    a.update(kw)
    return list(a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(prefix=24), -2), (dict(prefix=0), -2), (dict(B=32, prefix=48), -2), (dict(group=5), -2),
    (dict(dt=0), -3), (dict(np=1), -5), (dict(k_new=ctypes.c_void_p(16)), -1), (dict(po=None), -1),
])
def test_shared_prefix_rejects_bad_args_on_host(lib, kw, code):
    assert lib.pa_decode_shared_prefix(*_sp_args(**kw)) == code


def test_copy_blocks_and_append_reject_bad_args_on_host(lib):
    fake = ctypes.c_void_p(16)
    assert lib.pa_copy_blocks(fake, fake, 4, fake, fake, 4, fake, fake, 0, 2, 128, 16, 1, None) == 0  # no pairs
    assert lib.pa_copy_blocks(None, fake, 4, fake, fake, 4, fake, fake, 1, 2, 128, 16, 1, None) == -1
    assert lib.pa_copy_blocks(fake, fake, 4, fake, fake, 4, fake, fake, 1, 2, 128, 16, 9, None) == -3
    args = [fake, fake, None, fake, fake, fake, fake, 4, fake, 2, 8, 2, 128, 16, 10, ctypes.c_float(0.1), 1, None]
    assert lib.pa_decode_append(*args) == -1                       # k_new missing
    args[2] = ctypes.c_void_p(24)
    assert lib.pa_decode_append(*args) == -7                       # k_new misaligned


def test_binding_rejects_host_tensors_before_any_launch():
    """The Python layer refuses tensors the kernels could not address: no CPU fallback, no launch."""
    import torch

    import paged_kv_cache_475_b200 as pa
    q = torch.zeros(2, 8, 128, dtype=torch.float16)
    kc = torch.zeros(4, 2, 16, 128, dtype=torch.float16)
    bt = torch.zeros(2, 4, dtype=torch.int32)
    lens = torch.ones(2, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pa.pa_decode(torch.empty_like(q), q, kc, kc.clone(), bt, lens, 0.1)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pa.pa_reshape_and_cache(torch.zeros(1, 2, 128, dtype=torch.float16), torch.zeros(1, 2, 128, dtype=torch.float16),
                                kc, kc.clone(), torch.zeros(1, dtype=torch.int64))
    with pytest.raises(ValueError, match="pinned"):
        pa.pa_copy_blocks(kc, kc.clone(), kc, kc.clone(), torch.zeros(1, dtype=torch.int32),
                          torch.zeros(1, dtype=torch.int32))


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "pa.h"

int main(void) {
  int fails = 0;
  /* status strings, version, partition count */
  if (strcmp(pa_status_string(PA_OK), "PA_OK") != 0) fails++;
  if (pa_version() < 100) fails++;
  if (pa_splitkv_num_partitions(100000, 512) != 196) fails++;
  /* one workspace for part_o [4,32,196,128], part_m and part_l [4,32,196], each rounded to 256 B */
  if (pa_splitkv_workspace_bytes(4, 32, 128, 100000, 512) != (size_t)(4 * 32 * 196 * 128 * 4 + 2 * 100352))
    fails++;
  if (pa_splitkv_workspace_bytes(4, 0, 128, 100000, 512) != 0) fails++;
  /* host-side checks run before any device work */
  char fake[256];
  if (pa_decode(fake, fake, fake, fake, (const int32_t*)fake, 4, (const int32_t*)fake, 2, 8, 2, 96, 16, 10,
                0.1f, PA_F16, NULL) != PA_ERR_UNSUPPORTED) fails++;
  if (pa_decode(fake, NULL, fake, fake, (const int32_t*)fake, 4, (const int32_t*)fake, 2, 8, 2, 128, 16, 10,
                0.1f, PA_F16, NULL) != PA_ERR_NULL) fails++;
  if (pa_prefill_chunk(fake, fake, fake, fake, (const int32_t*)fake, 4, (const int32_t*)fake, 2, 8, 8, 2, 128,
                       16, 10, 0.1f, PA_F32, NULL) != PA_ERR_DTYPE) fails++;
  if (pa_reshape_and_cache(NULL, NULL, NULL, NULL, NULL, 0, 10, 8, 128, 16, PA_F16, NULL) != PA_OK) fails++;
  printf("fails=%d\n", fails);
  return fails;
}
"""


def test_header_compiles_as_c_and_links(lib, tmp_path):
    """The boundary is a C ABI: pa.h compiles as C99, a C program links libpa.so and gets the host-side
    status codes (no device work is started by these calls)."""
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi_check.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "abi_check"
    libdir = os.path.join(ROOT, "paged_kv_cache_475_b200")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                    str(exe), "-L", libdir, "-lpa", f"-Wl,-rpath,{libdir}"], check=True, capture_output=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "fails=0" in r.stdout
