"""Host-side checks of the boundary (no GPU compute): the C-ABI library
builds for sm_100a, loads, and exports every entry point include/nc.h
declares; the binding refuses to run without the library; the seeded input
generators behave as documented."""
import os
import re

import numpy as np
import pytest

from pretraining_step_b200 import binding, inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(nc_[a-z0-9_]+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol():
    from pretraining_step_b200 import build
    build.build()
    L = binding.lib()
    declared = _declared()
    assert len(declared) >= 25
    missing = [n for n in sorted(declared) if not hasattr(L, n)]
    assert not missing, missing


def test_binding_declares_a_signature_for_every_entry_point():
    """Every function of the C ABI is marshalled with declared argument and
    result types (ctypes would otherwise pass Python ints as C int)."""
    L = binding.lib()
    undeclared = [n for n in sorted(_declared()) if getattr(L, n).argtypes is None]
    assert not undeclared, undeclared


def test_status_strings():
    assert binding.status_string(binding.NC_OK) == "ok"
    assert binding.status_string(binding.NC_ERR_TIMEOUT) == "device wait timed out"
    assert binding.status_string(99) == "unknown"


def test_oracle_is_not_linked_by_the_product():
    import subprocess
    from pretraining_step_b200 import build
    out = subprocess.run(["nm", "-D", build.build()], capture_output=True, text=True).stdout
    assert "oc_" not in " ".join(l.split()[-1] for l in out.splitlines() if " T " in l)
    for dirpath, _, files in os.walk(os.path.join(ROOT, "pretraining_step_b200")):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "nc_oracle" not in src, f


def test_token_generator_range_and_shift():
    tok, tgt = inputs.token_batch(20, 4, 64)
    assert tok.dtype == np.int32 and tok.shape == (4, 64)
    assert tok.min() >= 0 and tok.max() < 32768
    assert np.array_equal(tok[:, 1:], tgt[:, :-1])
    a, _ = inputs.token_batch(20, 4, 64)
    b, _ = inputs.token_batch(21, 4, 64)
    assert np.array_equal(a, tok) and not np.array_equal(a, b)
    # V = 32768: ids are the top 15 bits of the SplitMix64 word.
    w = inputs.splitmix64(inputs.stream_key(20, inputs.STREAM_TOKENS) + np.uint64(0))
    assert tok[0, 0] == int(w) >> 49
    z, _ = inputs.zipf_token_batch(3, 8, 256)
    assert z.min() >= 0 and z.max() < 32768 and np.mean(z == 0) > 0.05


def test_bf16_rounding_is_exact_and_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, -2.5, 3.0e38], dtype=np.float32)
    r = inputs.round_to_bf16(x)
    assert r[0] == 1.0 and r[1] == 1.0 and r[2] == 1.0 + 2 ** -7 and r[3] == -2.5
    assert np.all((r.view(np.uint32) & 0xFFFF) == 0)


@pytest.mark.parametrize("depth,vocab,status", [(34, 512, "NC_ERR_INVALID_ARG"),   # 17 heads
                                                (3, 512, "NC_ERR_UNSUPPORTED"),    # odd depth
                                                (2, 12, "NC_ERR_INVALID_ARG")])    # vocab % 8
def test_init_rejects_unsupported_shapes(depth, vocab, status):
    """Shape validation runs before any CUDA call, so it is checked here."""
    with pytest.raises(binding.NcError) as e:
        binding.GPT(depth, vocab=vocab, seed=1)
    assert e.value.status == getattr(binding, status)


def test_adamw_step_refuses_a_null_handle():
    st = binding.lib().nc_adamw_step(None, None, 0.1, 0.1, 0.9, 0.95, 1e-8, 0.0)
    assert st == binding.NC_ERR_INVALID_ARG


@pytest.mark.parametrize("depth,n_kv_head", [(8, 3), (8, 5), (4, 4), (8, -1)])
def test_init_rejects_kv_heads_that_do_not_divide_the_heads(depth, n_kv_head):
    """depth 8 has 4 heads, depth 4 has 2: the KV-head count must divide them."""
    with pytest.raises(binding.NcError) as e:
        binding.GPT(depth, vocab=512, seed=1, n_kv_head=n_kv_head)
    assert e.value.status == binding.NC_ERR_INVALID_ARG


def test_window_pattern_repeats_over_layers():
    assert binding.window_pattern("SSSL", 6, 128) == [128, 128, 128, -1, 128, 128]
    assert binding.window_pattern("L", 2, 5) == [-1, -1]
    with pytest.raises(ValueError):
        binding.window_pattern("SXL", 4, 8)
    with pytest.raises(ValueError):
        binding.GPT(4, vocab=512, window=[1, 2, 3])


def test_step_graph_calls_refuse_a_null_handle():
    L = binding.lib()
    assert L.nc_step_replay(None) == binding.NC_ERR_INVALID_ARG
    assert L.nc_step_capture(None, None, None, 1, 1, None, None, 0.1, 0.9) == binding.NC_ERR_INVALID_ARG
