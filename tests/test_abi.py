"""The C ABI on the host (no GPU): the library loads, exports every symbol the
header declares, the ctypes mirror matches the C struct layout, and invalid
arguments are rejected synchronously before anything is launched."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

from differential_latent_attention_gdla_b200 import _abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdla.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_abi.LIB_PATH):
        build.build()
    return _abi.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gdla_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(names) == set(_abi.EXPORTED), names
    for n in names:
        assert hasattr(lib, n), n
    assert "sm_100a" in lib.gdla_build_info().decode()


def test_status_strings(lib):
    for code in range(6):
        assert lib.gdla_status_string(code)
    assert b"INVALID" in lib.gdla_status_string(_abi.GDLA_ERR_INVALID_ARG)


def _c_layout(struct: str, fields):
    prog = "#include <stdio.h>\n#include <stddef.h>\n#include \"gdla.h\"\nint main(void){\n"
    prog += f'printf("%zu\\n", sizeof({struct}));\n'
    for f in fields:
        prog += f'printf("%zu\\n", offsetof({struct}, {f}));\n'
    prog += "return 0;}\n"
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(prog)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout.split()
    return [int(x) for x in out]


@pytest.mark.parametrize("cls,cname", [(_abi.ExpandArgs, "gdla_expand_args"), (_abi.PrefillArgs, "gdla_prefill_args"),
                                       (_abi.AttendArgs, "gdla_attend_args"),
                                       (_abi.DecodeArgs, "gdla_decode_args"), (_abi.GatesArgs, "gdla_gates_args")])
def test_ctypes_mirror_matches_c_layout(cls, cname):
    fields = [f[0] for f in cls._fields_]
    got = [ctypes.sizeof(cls)] + [getattr(cls, f).offset for f in fields]
    assert got == _c_layout(cname, fields)


def good_prefill():
    a = _abi.PrefillArgs(2, 100, 512, 64, 16, 128, 128, 16, 3, _abi.GDLA_MASK_CAUSAL, 0, 0.0, 0.0, _abi.GDLA_BF16, 100)
    base = 0x10000000
    for i, f in enumerate(("c_kv", "gamma", "k_rope", "q", "w_ukv", "rope_cos", "rope_sin", "lam_logits",
                           "gate_logits", "out", "workspace")):
        setattr(a, f, base + i * 0x1000000)
    return a


def test_prefill_validation_rejects_before_launch(lib):
    def st(mut):
        a = good_prefill()
        a.workspace_bytes = lib.gdla_prefill_workspace_size(ctypes.byref(a))
        mut(a)
        return lib.gdla_prefill(ctypes.byref(a), None)

    E, U = _abi.GDLA_ERR_INVALID_ARG, _abi.GDLA_ERR_UNSUPPORTED
    assert st(lambda a: setattr(a, "B", 0)) == E
    assert st(lambda a: setattr(a, "L", 0)) == E
    assert st(lambda a: setattr(a, "q", 0)) == E                      # NULL
    assert st(lambda a: setattr(a, "q", 0x10000008)) == E             # misaligned
    assert st(lambda a: setattr(a, "workspace", a.workspace + 16)) == E  # not 256-aligned
    assert st(lambda a: setattr(a, "workspace_bytes", a.workspace_bytes - 1)) == E
    assert st(lambda a: setattr(a, "rope_max_pos", 99)) == E
    assert st(lambda a: (setattr(a, "mask", _abi.GDLA_MASK_SLIDING), setattr(a, "window", 0))) == E
    assert st(lambda a: setattr(a, "mask", 7)) == E
    assert st(lambda a: setattr(a, "dtype", 5)) == E
    assert st(lambda a: setattr(a, "n_noise", 8)) == U                # n_noise != n_kv
    assert st(lambda a: setattr(a, "g", 9)) == U
    assert st(lambda a: setattr(a, "d_nope", 96)) == U
    assert st(lambda a: setattr(a, "d_c", 300)) == U
    assert st(lambda a: setattr(a, "cache_c_hat", 0x20000004)) == E   # optional but misaligned
    assert lib.gdla_prefill(None, None) == E


def test_prefill_accepts_eighty_heads(lib):
    # the report's attention shape (16 KV heads, g = 4: 64 signal + 16 noise heads) is a
    # valid prefill; sizing needs no launch
    a = good_prefill()
    a.g = 4
    assert lib.gdla_prefill_workspace_size(ctypes.byref(a)) > 0


def test_prefill_workspace_size_is_monotone(lib):
    a = good_prefill()
    s1 = lib.gdla_prefill_workspace_size(ctypes.byref(a))
    a.L = 200
    s2 = lib.gdla_prefill_workspace_size(ctypes.byref(a))
    assert s2 > s1 > 2 * 100 * 16 * 256 * 2
    assert s1 % 256 == 0


def test_decode_validation_rejects_before_launch(lib):
    def good():
        a = _abi.DecodeArgs(4, 1000, 512, 64, 16, 128, 128, 16, 2, _abi.GDLA_MASK_CAUSAL, 0, 0.0, _abi.GDLA_BF16,
                            1000)
        base = 0x10000000
        for i, f in enumerate(("seqlens", "c_cache", "kr_cache", "q", "w_ukv", "rope_cos", "rope_sin", "lam_logits",
                               "gate_logits", "out", "workspace")):
            setattr(a, f, base + i * 0x1000000)
        a.workspace_bytes = lib.gdla_decode_workspace_size(ctypes.byref(a))
        return a

    E, U = _abi.GDLA_ERR_INVALID_ARG, _abi.GDLA_ERR_UNSUPPORTED
    for mut, want in ((lambda a: setattr(a, "B", 0), E), (lambda a: setattr(a, "c_cache", 0), E),
                      (lambda a: setattr(a, "workspace_bytes", 1024), E), (lambda a: setattr(a, "rope_max_pos", 10), E),
                      (lambda a: setattr(a, "n_noise", 4), U), (lambda a: setattr(a, "d_rope", 48), U),
                      # 16 x 5 = 80 query heads: the tensor-core (bf16) decode takes them in two head
                      # groups; the CUDA-core (fp32) decode holds at most 64 heads per block
                      (lambda a: (setattr(a, "g", 4), setattr(a, "dtype", _abi.GDLA_FP32)), U),
                      (lambda a: (setattr(a, "mask", 1), setattr(a, "window", -3)), E)):
        a = good()
        mut(a)
        assert lib.gdla_decode(ctypes.byref(a), None) == want
    assert lib.gdla_decode_workspace_size(ctypes.byref(good())) > 4 * 48 * 512 * 4


def test_expand_validation(lib):
    a = _abi.ExpandArgs(1, 10, 512, 64, 16, 128, 128, _abi.GDLA_BF16, 0.0, 5)
    assert lib.gdla_latent_expand(ctypes.byref(a), None) == _abi.GDLA_ERR_INVALID_ARG  # table too short
    a.rope_max_pos = 10
    assert lib.gdla_latent_expand(ctypes.byref(a), None) == _abi.GDLA_ERR_INVALID_ARG  # NULL pointers


def good_attend():
    a = _abi.AttendArgs(2, 300, 64, 16, 128, 128, 16, 3, _abi.GDLA_MASK_CAUSAL, 0, 0.0, _abi.GDLA_BF16, 300)
    base = 0x10000000
    for i, f in enumerate(("q", "kv", "k_rope_rot", "rope_cos", "rope_sin", "lam_logits", "gate_logits", "out",
                           "workspace")):
        setattr(a, f, base + i * 0x1000000)
    a.workspace_bytes = 256
    return a


def test_attend_query_block_validation(lib):
    # the query block must lie inside the L key positions; q_len == 0 means all rows
    E = _abi.GDLA_ERR_INVALID_ARG
    for q_len, q_start in ((-1, 0), (10, -1), (0, 5), (301, 0), (200, 101), (1, 300)):
        a = good_attend()
        a.q_len, a.q_start = q_len, q_start
        assert lib.gdla_attend(ctypes.byref(a), None) == E, (q_len, q_start)


def test_prefill_host_validation_rejects_before_launch(lib):
    def st(mut, chunk=256):
        a = good_prefill()
        a.workspace_bytes = lib.gdla_prefill_host_workspace_size(ctypes.byref(a), chunk)
        mut(a)
        return lib.gdla_prefill_host(ctypes.byref(a), chunk, None)

    E, U = _abi.GDLA_ERR_INVALID_ARG, _abi.GDLA_ERR_UNSUPPORTED
    assert st(lambda a: setattr(a, "q", 0)) == E                       # host input NULL
    assert st(lambda a: setattr(a, "out", 0)) == E                     # host output NULL
    assert st(lambda a: setattr(a, "gamma", 0x10000004)) == E          # device parameter misaligned
    assert st(lambda a: setattr(a, "workspace", a.workspace + 16)) == E
    assert st(lambda a: setattr(a, "workspace_bytes", a.workspace_bytes - 1)) == E
    assert st(lambda a: setattr(a, "rope_max_pos", 99)) == E
    assert st(lambda a: setattr(a, "g", 9)) == U
    assert lib.gdla_prefill_host(None, 0, None) == E


def test_prefill_host_workspace_size(lib):
    # the prefill workspace, device copies of c_kv and k_rope, and eight chunk-sized
    # staging slots for q, lambda, gate and Y
    a = good_prefill()  # B=2, L=100, 16 KV heads, g=3: 64 query heads
    base = lib.gdla_prefill_workspace_size(ctypes.byref(a))
    latent = 2 * 100 * (512 + 64) * 2
    s64 = lib.gdla_prefill_host_workspace_size(ctypes.byref(a), 64)
    per_tok = 64 * 192 * 2 + 48 * 4 + 2 * 48 * 128 * 2  # q, lambda, gate + Y
    assert s64 >= base + latent + 8 * 64 * per_tok
    assert s64 <= base + latent + 2 * 256 + 8 * (64 * per_tok + 4 * 256)
    assert s64 % 256 == 0
    # chunks longer than the sequence (and the default) clamp to L
    s_full = lib.gdla_prefill_host_workspace_size(ctypes.byref(a), 100)
    assert lib.gdla_prefill_host_workspace_size(ctypes.byref(a), 5000) == s_full
    assert lib.gdla_prefill_host_workspace_size(ctypes.byref(a), 0) == s_full
    assert s_full > s64
    assert lib.gdla_prefill_host_workspace_size(None, 64) == 0


def good_gates():
    a = _abi.GatesArgs(2, 100, 1536, 2048, 48, 128, _abi.GDLA_BF16, 0.0)
    base = 0x10000000
    for i, f in enumerate(("c_q", "gamma_q", "w_g", "x", "w_lambda", "gate_logits", "lam_logits", "workspace")):
        setattr(a, f, base + i * 0x1000000)
    a.workspace_bytes = lib_gates_ws(a)
    return a


def lib_gates_ws(a):
    return _abi.load().gdla_gates_workspace_size(ctypes.byref(a))


def test_gates_workspace_size(lib):
    a = good_gates()
    assert lib.gdla_gates_workspace_size(ctypes.byref(a)) == 256 + 2 * 100 * 1536 * 2  # status + c_hat_q
    a.c_q = None  # lambda only: the status word alone
    assert lib.gdla_gates_workspace_size(ctypes.byref(a)) == 256
    assert lib.gdla_gates_workspace_size(None) == 0


def test_gates_validation_rejects_before_launch(lib):
    E = _abi.GDLA_ERR_INVALID_ARG

    def st(mut):
        a = good_gates()
        mut(a)
        return lib.gdla_gates(ctypes.byref(a), None)

    assert st(lambda a: setattr(a, "B", 0)) == E
    assert st(lambda a: setattr(a, "n_signal", 0)) == E
    assert st(lambda a: setattr(a, "dtype", 3)) == E
    assert st(lambda a: setattr(a, "w_g", 0)) == E                     # gate requested without W_G
    assert st(lambda a: setattr(a, "gate_logits", 0x10000004)) == E    # misaligned output
    assert st(lambda a: setattr(a, "w_lambda", 0)) == E                # lambda requested without W_lambda
    assert st(lambda a: setattr(a, "d_x", 0)) == E
    assert st(lambda a: setattr(a, "workspace", a.workspace + 16)) == E
    assert st(lambda a: setattr(a, "workspace_bytes", a.workspace_bytes - 1)) == E
    assert lib.gdla_gates(None, None) == E


def test_rope_table_builders_reject_bad_arguments_and_write_nothing(lib):
    fp = ctypes.POINTER(ctypes.c_float)
    buf = (ctypes.c_float * 64)(*([7.0] * 64))
    p = ctypes.cast(buf, fp)
    E = _abi.GDLA_ERR_INVALID_ARG
    assert lib.gdla_rope_tables(0, 8, 10000.0, p, p) == E
    assert lib.gdla_rope_tables(4, 7, 10000.0, p, p) == E
    assert lib.gdla_rope_tables(4, 8, 1.0, p, p) == E
    assert lib.gdla_rope_tables(4, 8, 10000.0, None, p) == E
    assert lib.gdla_yarn_rope_tables(4, 8, 10000.0, 0.0, 64, 32.0, 1.0, p, p) == E
    assert lib.gdla_yarn_rope_tables(4, 8, 10000.0, 4.0, 0, 32.0, 1.0, p, p) == E
    assert lib.gdla_yarn_rope_tables(4, 8, 10000.0, 4.0, 64, 0.0, 1.0, p, p) == E
    assert list(buf) == [7.0] * 64
    assert lib.gdla_rope_tables(4, 8, 10000.0, p, ctypes.cast(ctypes.byref(buf, 64), fp)) == _abi.GDLA_OK
    assert buf[0] == 1.0 and buf[16] == 0.0  # position 0: cos 1, sin 0
    assert lib.gdla_yarn_mscale(1.0) == 1.0 and lib.gdla_yarn_mscale(0.5) == 1.0
