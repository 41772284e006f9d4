"""The C ABI on the host: the library loads, exports every entry point the
header declares, and rejects bad arguments before touching a GPU."""
import ctypes
import os
import re

import pytest

from parameterized_local_linear_b200 import binding, build

INCLUDE = os.path.join(os.path.dirname(build.PKG), "include")
HEADER = os.path.join(INCLUDE, "parallax.h")
HEADERS = sorted(os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h"))

OK, ENULL, ESHAPE, EHEAD, EDTYPE, EALIGN, EWS, ESPLITS = 0, -1, -2, -3, -4, -5, -6, -7


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load_library()


def declared_functions():
    names = set()
    for h in HEADERS:
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\b(parallax_\w+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("parallax_decode", "parallax_softmax_decode", "parallax_decode_phase",
                     "parallax_decode_workspace_bytes", "parallax_choose_splits",
                     "parallax_status_string", "parallax_workspace_status"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in parallax.h but not exported"


def test_header_compiles_as_c(tmp_path):
    src = tmp_path / "t.c"
    src.write_text("".join(f'#include "{os.path.basename(h)}"\n' for h in HEADERS) +
                   "int main(void){return PARALLAX_OK;}\n")
    import subprocess
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER),
                    "-c", str(src), "-o", str(tmp_path / "t.o")], check=True)


def test_status_strings(lib):
    for code in range(-11, 1):
        s = binding.parallax_status_string(code)
        assert s and s != "unknown status"
    assert binding.parallax_status_string(-99) == "unknown status"


def test_choose_splits_host_only(lib):
    # explicit SM count: pure host arithmetic
    assert lib.parallax_choose_splits(1, 8, 4096, 148) == 148     # one CTA per SM
    assert lib.parallax_choose_splits(1, 8, 1024, 148) == 64      # 8192 keys / 128
    assert lib.parallax_choose_splits(2048, 8, 4096, 148) == 148
    assert lib.parallax_choose_splits(1, 1, 1, 148) == 1
    assert lib.parallax_choose_splits(2, 2, 128, 148) == 4  # 512 keys / 128
    assert lib.parallax_choose_splits(0, 8, 4096, 148) == ESHAPE
    # the default a call with num_splits = 0 uses: the generic kernel's finer count
    # for fp32 inputs or large groups (keys / 64), else the count above
    f = lib.parallax_default_splits
    bf16, f32 = 0, 1
    assert f(2, 4, 2, 128, bf16, 1, 148) == 4     # TMA kernel: 512 keys / 128
    assert f(2, 4, 2, 128, f32, 1, 148) == 8      # generic (fp32): 512 keys / 64
    assert f(1, 16, 2, 1024, bf16, 1, 148) == 32  # G = 8 with the probe: generic
    assert f(1, 16, 2, 1024, bf16, 0, 148) == 16  # G = 8 without: TMA kernel
    assert f(1, 16, 8, 4096, f32, 1, 148) == 148  # capped at one CTA per SM
    assert f(1, 12, 8, 4096, bf16, 1, 148) == ESHAPE


def test_workspace_bytes_host_only(lib):
    # 256-byte header + 2 records per split and query head of a group
    G, D, P = 2, 128, 10
    want = 256 + 2 * P * G * (4 + 2 * D) * 4
    assert lib.parallax_decode_workspace_bytes(1, 16, 8, 128, 4096, P) == want
    assert lib.parallax_decode_workspace_bytes(1, 16, 8, 96, 4096, P) == 0  # D
    assert lib.parallax_decode_workspace_bytes(1, 15, 8, 128, 4096, P) == 0  # Hq % Hkv
    assert lib.parallax_decode_workspace_bytes(1, 16, 8, 128, 4096, -1) == 0


def _call(lib, **kw):
    a = dict(q=16, r=16, k=16, v=16, n=16, out=16, B=1, Hq=16, Hkv=8, D=128, scale=0.1,
             stream=None, Lmax=64, ind=0, outd=0, splits=4, ws=16, wsb=1 << 20)
    a.update(kw)
    return lib.parallax_decode(a["q"], a["r"], a["k"], a["v"], a["n"], a["out"], a["B"], a["Hq"],
                               a["Hkv"], a["D"], ctypes.c_float(a["scale"]), a["stream"],
                               a["Lmax"], a["ind"], a["outd"], a["splits"], a["ws"], a["wsb"])


def test_argument_errors_before_launch(lib):
    # Fake, aligned, never dereferenced addresses: each call fails validation
    # on the host, so nothing reaches the device.
    assert _call(lib, q=None) == ENULL
    assert _call(lib, r=None) == ENULL
    assert _call(lib, ws=None) == ENULL
    assert _call(lib, Hq=12) == ESHAPE
    assert _call(lib, B=0) == ESHAPE
    assert _call(lib, Lmax=0) == ESHAPE
    assert _call(lib, D=96) == EHEAD
    assert _call(lib, ind=2) == EDTYPE
    assert _call(lib, outd=-1) == EDTYPE
    assert _call(lib, k=24) == EALIGN
    assert _call(lib, out=8) == EALIGN
    assert _call(lib, n=18) == EALIGN
    assert _call(lib, splits=-1) == ESPLITS
    assert _call(lib, splits=65537) == ESPLITS
    assert _call(lib, wsb=100) == EWS  # explicit splits: sized on the host


def test_softmax_decode_does_not_need_r(lib):
    rc = lib.parallax_softmax_decode(16, 16, 16, 16, 16, 1, 16, 8, 128, ctypes.c_float(0.1),
                                     None, 64, 0, 0, 4, 16, 100)
    assert rc == EWS  # got past the pointer checks without r


def test_stall_hook_rejects_bad_timeout(lib):
    fn = lib.parallax_testing_decode_stalled
    fn.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int] * 4 + [ctypes.c_float, ctypes.c_void_p,
                                                                ctypes.c_int, ctypes.c_int,
                                                                ctypes.c_void_p, ctypes.c_size_t,
                                                                ctypes.c_int]
    assert fn(16, 16, 16, 16, 16, 16, 1, 16, 8, 128, 0.1, None, 64, 4, 16, 1 << 20, 0) == ESHAPE
    assert fn(16, 16, 16, 16, 16, 16, 1, 16, 8, 128, 0.1, None, 64, 4, 16, 1 << 20, 20000) == ESHAPE


def test_phase_selector(lib):
    rc = lib.parallax_decode_phase(3, 1, 16, 16, 16, 16, 16, 16, 1, 16, 8, 128,
                                   ctypes.c_float(0.1), None, 64, 0, 0, 4, 16, 1 << 20)
    assert rc == -10


def test_prefill_argument_errors_before_launch(lib):
    fn = lib.parallax_prefill
    fn.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 5 + [ctypes.c_float, ctypes.c_int,
                                                                ctypes.c_void_p, ctypes.c_int,
                                                                ctypes.c_void_p, ctypes.c_size_t]
    fn.restype = ctypes.c_int

    def call(q=16, out=16, B=1, Hq=4, Hkv=2, L=64, D=128, scale=0.1, outd=0, ws=16, wsb=256):
        return fn(q, 16, 16, 16, out, B, Hq, Hkv, L, D, scale, 1, None, outd, ws, wsb)

    assert call(q=None) == ENULL
    assert call(ws=None) == ENULL
    assert call(Hq=3) == ESHAPE
    assert call(L=0) == ESHAPE
    assert call(scale=0.0) == ESHAPE  # the softmax temperature must be positive
    assert call(scale=-0.1) == ESHAPE
    assert call(scale=float("inf")) == ESHAPE
    assert call(scale=float("nan")) == ESHAPE
    assert call(D=96) == EHEAD
    assert call(outd=2) == EDTYPE
    assert call(out=8) == EALIGN
    assert call(wsb=100) == EWS


def test_split_env_override():
    """PARALLAX_SPLITS replaces the split heuristic (read once per process)."""
    import os
    import subprocess
    import sys
    code = ("import ctypes, sys; lib = ctypes.CDLL(sys.argv[1]); "
            "print(lib.parallax_choose_splits(1, 8, 4096, 148))")
    path = binding.library_path()
    run = lambda env: subprocess.run([sys.executable, "-c", code, path], capture_output=True,
                                     text=True, env=env, check=True).stdout.strip()
    base = {k: v for k, v in os.environ.items() if k != "PARALLAX_SPLITS"}
    assert run(base) == "148"
    assert run({**base, "PARALLAX_SPLITS": "37"}) == "37"
    assert run({**base, "PARALLAX_SPLITS": "junk"}) == "148"


def test_prefill_workspace_bytes(lib):
    """Header 256 B (padded to 1024), the fp16 copy of V, 4 bytes per (kv item,
    64-key block); 0 for arguments outside the supported shapes."""
    f = binding.parallax_prefill_workspace_bytes
    B, L, Hkv, D = 4, 4096, 8, 128
    v16 = B * L * Hkv * D * 2
    assert f(B, L, Hkv, D) == 1024 + v16 + B * Hkv * (L // 64) * 4
    # packed: one item per kv head over all tokens; a partial last block counts
    assert f(1, 9991, 8, 64) == 1024 + (9991 * 8 * 64 * 2 + 255) // 256 * 256 + 8 * 157 * 4
    for bad in ((0, 1, 1, 64), (1, 0, 1, 64), (1, 1, 0, 64), (1, 1, 1, 96)):
        assert f(*bad) == 0
