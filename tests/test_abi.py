"""C-ABI library (no GPU): it builds, loads, exports every declared symbol, and
rejects bad arguments on the host before touching a device."""
import ctypes
import glob
import os
import re

import pytest

import sparse_attention_token_index_b200 as dsa
from sparse_attention_token_index_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    B.build()
    return dsa.lib()


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        txt = open(h).read()
        txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
        names |= set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(dsa_\w+)\s*\(", txt, flags=re.M))
    return names


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert set(dsa.EXPORTED_SYMBOLS) <= names


def test_version_and_status_strings(L):
    assert L.dsa_version() == 100
    assert L.dsa_status_string(0) == b"ok"
    for code in (-1, -2, -3, -4, -5, -6, -7):
        assert L.dsa_status_string(code) != b"unknown status"


def test_host_validation_before_device(L):
    n = ctypes.c_size_t(0)
    f = L.dsa_index_dense
    ok_ptr = ctypes.c_void_p(4096)
    # null Q
    assert f(None, ok_ptr, ok_ptr, None, 4, 4, 64, 128, 0, 2, 0, 0, ok_ptr, ok_ptr, ok_ptr, 1 << 20, None) == -1
    # k out of range
    assert f(ok_ptr, ok_ptr, ok_ptr, None, 4, 4, 64, 128, 0, 0, 0, 0, ok_ptr, ok_ptr, ok_ptr, 1 << 20, None) == -1
    # causal range past the keys
    assert f(ok_ptr, ok_ptr, ok_ptr, None, 4, 4, 64, 128, 1, 2, 0, 0, ok_ptr, ok_ptr, ok_ptr, 1 << 20, None) == -1
    # unsupported shape (H * d too large)
    assert f(ok_ptr, ok_ptr, ok_ptr, None, 4, 4, 128, 256, 0, 2, 0, 0, ok_ptr, ok_ptr, ok_ptr, 1 << 20, None) == -2
    # misaligned Q
    assert f(ctypes.c_void_p(4100), ok_ptr, ok_ptr, None, 4, 4, 64, 128, 0, 2, 0, 0, ok_ptr, ok_ptr, ok_ptr,
             1 << 20, None) == -1
    # fp8 keys need a scale
    assert f(ok_ptr, ok_ptr, ok_ptr, None, 4, 4, 64, 128, 0, 2, 0, 2, ok_ptr, ok_ptr, ok_ptr, 1 << 20, None) == -1
    # group: bank smaller than k
    g = L.dsa_index_group
    assert g(ok_ptr, ok_ptr, ok_ptr, None, 8, 8, 64, 128, 0, 4, 2, 2, 0, 0, 0, ok_ptr, ok_ptr, None, None, None,
             None, ok_ptr, 1 << 20, None) == -1
    # workspace-size query rejects a null output pointer
    assert L.dsa_index_dense_workspace_size(4, 4, 64, 128, 2, 0, 0, None) == -1
    assert n.value == 0


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(2, 64, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        dsa.dsa_index_dense(q, torch.zeros(2, 64), torch.zeros(4, 128, dtype=torch.bfloat16), 2)


def test_kernel_timer_host_checks(L):
    ms, n = ctypes.c_float(0.0), ctypes.c_int(0)
    # stop while disarmed, null outputs, and out-of-range counts are refused
    # before any CUDA call
    assert L.dsa_kernel_timer_stop(ctypes.byref(ms), ctypes.byref(n)) == -1
    assert L.dsa_kernel_timer_stop(None, None) == -1
    assert L.dsa_kernel_timer_start(0) == -1
    assert L.dsa_kernel_timer_start((1 << 20) + 1) == -1


def test_decode_host_checks(L):
    ok = ctypes.c_void_p(4096)
    f = L.dsa_index_decode
    # max_keys above total_keys
    assert f(ok, ok, ok, None, ok, ok, 1, 2, 100, 101, 64, 128, 16, 0, 0, ok, ok, ok, 1 << 20, None) == -1
    # more keys than 32-bit TMA row coordinates reach (tensor-core shape)
    assert f(ok, ok, ok, None, ok, ok, 1, 2, 1 << 31, 1 << 20, 64, 128, 16, 0, 0, ok, ok, ok, 1 << 20, None) == -2


def test_comparator_and_group_host_checks(L):
    ok = ctypes.c_void_p(4096)
    n = ctypes.c_size_t(0)
    # block routing: null Q, zero blocks
    f = L.dsa_index_block_routed
    assert f(None, ok, ok, None, 8, 256, 64, 128, 248, 4, 2, 0, 0, ok, ok, None, None, ok, 1 << 20, None) == -1
    assert f(ok, ok, ok, None, 8, 256, 64, 128, 248, 4, 0, 0, 0, ok, ok, None, None, ok, 1 << 20, None) == -1
    # inverted file: more clusters than keys, d not a multiple of 32
    assert L.dsa_ivf_index_size(100, 128, 200, ctypes.byref(n)) == -1
    assert L.dsa_ivf_index_size(100, 100, 10, ctypes.byref(n)) == -1
    assert L.dsa_ivf_index_size(100, 128, 10, ctypes.byref(n)) == 0 and n.value > 100 * 128 * 2
    # routed query: more probes than clusters
    g = L.dsa_index_ivf_routed
    assert g(ok, ok, ok, None, 8, 256, 64, 128, 248, 4, 10, 11, 4, 0, 0, ok, ok, None, ok, 1 << 20, None) == -1
    # decode group: bank smaller than k, unknown mode
    h = L.dsa_index_decode_group
    assert h(ok, ok, ok, None, ok, ok, 1, 2, 100, 100, 64, 128, 16, 8, 0, 0, 0, ok, ok, None, None, None, None, ok,
             1 << 20, None) == -1
    assert h(ok, ok, ok, None, ok, ok, 1, 2, 100, 100, 64, 128, 16, 32, 7, 0, 0, ok, ok, None, None, None, None, ok,
             1 << 20, None) == -1
    # group: unknown mode
    gg = L.dsa_index_group
    assert gg(ok, ok, ok, None, 8, 8, 64, 128, 0, 4, 2, 8, 7, 0, 0, ok, ok, None, None, None, None, ok, 1 << 20,
              None) == -1


def test_empty_calls_need_no_device(L):
    # no query rows: the shape arguments are checked, nothing is launched, no
    # device is touched, and NULL tensor pointers are accepted
    n = ctypes.c_size_t(0)
    assert L.dsa_index_dense_workspace_size(0, 10, 64, 128, 4, 0, 0, ctypes.byref(n)) == 0 and n.value == 256
    assert L.dsa_index_dense(None, None, None, None, 0, 10, 64, 128, 10, 4, 0, 0, None, None, None, 0, None) == 0
    assert L.dsa_index_dense(None, None, None, None, 0, 0, 64, 128, 0, 4, 0, 0, None, None, None, 0, None) == 0
    assert L.dsa_index_group(None, None, None, None, 0, 10, 64, 128, 10, 4, 8, 16, 0, 0, 0, None, None, None, None,
                             None, None, None, 0, None) == 0
    assert L.dsa_index_decode(None, None, None, None, None, None, 0, 0, 0, 0, 64, 128, 4, 0, 0, None, None, None, 0,
                              None) == 0
    assert L.dsa_index_decode_group(None, None, None, None, None, None, 0, 0, 0, 0, 64, 128, 4, 16, 0, 0, 0, None,
                                    None, None, None, None, None, None, 0, None) == 0
    assert L.dsa_index_dense_static(None, None, None, 0, 10, 64, 128, 10, 4, None, None, None) == 0
    assert L.dsa_index_dense_host(None, None, None, None, 0, 10, 64, 128, 10, 4, 0, 0, 0, None, None, None, 0,
                                  None) == 0
    assert L.dsa_index_decode_host(None, None, None, None, None, None, 0, 0, 0, 0, 64, 128, 4, 0, 0, None, None, None,
                                   0, None) == 0
    # still checked: k, q_pos0 against the keys, the group arguments, decode totals
    assert L.dsa_index_dense(None, None, None, None, 0, 10, 64, 128, 10, 0, 0, 0, None, None, None, 0, None) == -1
    assert L.dsa_index_dense(None, None, None, None, 0, 10, 64, 128, 11, 4, 0, 0, None, None, None, 0, None) == -1
    assert L.dsa_index_group(None, None, None, None, 0, 10, 64, 128, 10, 16, 8, 8, 0, 0, 0, None, None, None, None,
                             None, None, None, 0, None) == -1
    assert L.dsa_index_decode(None, None, None, None, None, None, 0, 1, 0, 0, 64, 128, 4, 0, 0, None, None, None, 0,
                              None) == -1


def _declared_params():
    """name -> list of parameter type strings, from the header's prototypes."""
    out = {}
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        txt = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        for m in re.finditer(r"(?:const\s+)?\w+\s*\*?\s*(dsa_\w+)\s*\(([^)]*)\)\s*;", txt):
            params = [p.strip() for p in m.group(2).split(",") if p.strip() and p.strip() != "void"]
            out[m.group(1)] = params
    return out


def test_binding_prototypes_match_the_header():
    # every ctypes prototype has the header's parameter count, and each
    # pointer / 64-bit / 32-bit slot the matching ctypes kind
    import ctypes as C
    from sparse_attention_token_index_b200 import _binding as Bd
    decl = _declared_params()
    for name, (_, argtypes) in Bd._SIGS.items():
        assert name in decl, name
        params = decl[name]
        assert len(params) == len(argtypes), (name, len(params), len(argtypes))
        for p, t in zip(params, argtypes):
            if "*" in p:
                assert t in (C.c_void_p,) or issubclass(t, C._Pointer), (name, p, t)
            elif re.match(r"(const\s+)?(int64_t|size_t)\b", p):
                assert t in (C.c_int64, C.c_size_t), (name, p, t)
            elif re.match(r"unsigned\s+int\b", p):
                assert t is C.c_uint, (name, p, t)
            else:
                assert t is C.c_int, (name, p, t)


def test_plain_c_program_links_and_calls(tmp_path, L):
    # the header is C (not only C++), and a C program links against the
    # library and calls it: version, status text, and empty calls (no device)
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(r"""
#include <stdio.h>
#include <string.h>
#include "dsa_index.h"
int main(void) {
  size_t n = 0;
  if (dsa_version() != 100) return 1;
  if (strcmp(dsa_status_string(DSA_ERR_INVALID_ARG), "invalid argument") != 0) return 2;
  if (dsa_index_dense_workspace_size(0, 16, 64, 128, 8, DSA_DTYPE_BF16, DSA_DTYPE_BF16, &n) != DSA_OK || n != 256)
    return 3;
  if (dsa_index_dense(NULL, NULL, NULL, NULL, 0, 16, 64, 128, 16, 8, DSA_DTYPE_BF16, DSA_DTYPE_BF16, NULL, NULL,
                      NULL, 0, NULL) != DSA_OK)
    return 4;
  if (dsa_index_dense(NULL, NULL, NULL, NULL, 0, 16, 64, 128, 16, 0, DSA_DTYPE_BF16, DSA_DTYPE_BF16, NULL, NULL,
                      NULL, 0, NULL) != DSA_ERR_INVALID_ARG)
    return 5;
  puts("c abi ok");
  return 0;
}
""")
    lib = dsa.lib_path
    exe = tmp_path / "abi"
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                        str(exe), lib, "-Wl,-rpath," + os.path.dirname(lib)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and "c abi ok" in r.stdout, (r.returncode, r.stdout, r.stderr)


def test_binding_rejects_wrong_output_buffers():
    # caller-supplied outputs are checked before the library could write past them
    import torch
    from sparse_attention_token_index_b200 import _binding as Bd
    ok = (torch.empty((4, 8), dtype=torch.int32), torch.empty((4, 8), dtype=torch.float32))
    assert Bd._host_outputs(4, 8, ok) is ok
    with pytest.raises(ValueError):
        Bd._host_outputs(4, 8, (torch.empty((4, 7), dtype=torch.int32), torch.empty((4, 8), dtype=torch.float32)))
    with pytest.raises(TypeError):
        Bd._host_outputs(4, 8, (torch.empty((4, 8), dtype=torch.int64), torch.empty((4, 8), dtype=torch.float32)))


def test_binding_rejects_mismatched_shapes_before_any_call():
    # shapes the library cannot see through its pointers are checked first
    import torch
    q = torch.zeros((4, 64, 128), dtype=torch.bfloat16)
    w = torch.zeros((4, 64), dtype=torch.float32)
    K = torch.zeros((16, 128), dtype=torch.bfloat16)
    for args, kw in [((q, w[:, :32], K, 2), {}),                       # w not [T, H]
                     ((q, w.double(), K, 2), {}),                      # w not float32
                     ((q, w, K[:, :64], 2), {}),                       # K not [N, d]
                     ((q, w, K.to(torch.uint8), 2), {"K_scale": torch.zeros(15)})]:  # scales not [N]
        with pytest.raises(ValueError):
            dsa.dsa_index_dense(*args, **kw)
        with pytest.raises(ValueError):
            dsa.dsa_index_dense_host(*args, **kw)
    with pytest.raises(ValueError):
        dsa.dsa_index_decode_host(q, w, K, 2, torch.tensor([0, 8, 16]), torch.tensor([0, 4]))


def _offsets_cases():
    # (k_offsets, q_offsets, max_keys): each breaks one rule of the decode batch
    return [
        ([0, 8, 16], [0, 2, 3], 8),      # q_offsets[B] is not the 4 query rows
        ([1, 8, 16], [0, 2, 4], 8),      # k_offsets does not start at 0
        ([0, 8, 17], [0, 2, 4], 9),      # k_offsets[B] beyond K's 16 rows
        ([0, 8, 8], [0, 2, 4], 8),       # an empty cache (N_b = 0)
        ([0, 12, 16], [0, 2, 4], 8),     # N_b above max_keys
        ([0, 8, 16], [0, 0, 4], 8),      # a sequence without new queries
        ([0, 1, 16], [0, 2, 4], 15),     # m_b > N_b
        ([0, 8, 16], [0, 5, 4], 8),      # m_b above 4 (and decreasing offsets)
    ]


def test_binding_checks_host_decode_offsets():
    import torch
    from sparse_attention_token_index_b200 import _binding as Bd
    q = torch.zeros((4, 64, 128), dtype=torch.bfloat16)
    K = torch.zeros((16, 128), dtype=torch.bfloat16)
    for ko, qo, mk in _offsets_cases():
        with pytest.raises(ValueError):
            Bd._decode_offsets(q, K, torch.tensor(ko), torch.tensor(qo, dtype=torch.int32), mk, ko[-1])
    # a valid batch passes, sizes taken from the offsets when not given
    ko, qo, mk, tk = Bd._decode_offsets(q, K, torch.tensor([0, 8, 16]), torch.tensor([0, 2, 4], dtype=torch.int32),
                                        None, None)
    assert (mk, tk) == (8, 16)
    with pytest.raises(ValueError):   # total_keys beyond K's rows, even for device-side offsets
        Bd._decode_offsets(q, K, torch.tensor([0, 8, 16]), torch.tensor([0, 2, 4], dtype=torch.int32), 8, 17)


def test_host_decode_entry_checks_every_offset(L):
    # the host-buffer decode call reads its offsets on the host and rejects a
    # bad batch before any device work
    ok = ctypes.c_void_p(4096)
    for ko, qo, mk in _offsets_cases():
        if ko[-1] == 17:
            continue  # K's row count is the binding's to check: the C call sees total_keys only
        kk = (ctypes.c_int64 * len(ko))(*ko)
        qq = (ctypes.c_int32 * len(qo))(*qo)
        r = L.dsa_index_decode_host(ok, ok, ok, None, ctypes.cast(kk, ctypes.c_void_p),
                                    ctypes.cast(qq, ctypes.c_void_p), 2, 4, ko[-1], mk, 64, 128, 4, 0, 0, ok, ok, ok,
                                    1 << 30, None)
        assert r == -1, (ko, qo, mk, r)
