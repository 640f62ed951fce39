"""CPU checks of the C-ABI library: it loads, exports every symbol the
header declares, validates arguments before touching CUDA, computes the
slab/ring layout, and its NF4 codebook equals the oracle's bit for bit."""
import os
import re

import numpy as np
import pytest

from host_streamed_nf4_b200 import hsnf4, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hsnf4.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?(?:int|size_t|char|uint64_t)\s*\**\s*([a-z0-9_]+)\s*\(",
                                 src, flags=re.M)))


def test_library_exports_every_declared_symbol():
    L = hsnf4.lib()
    names = _declared()
    assert len(names) >= 20
    for n in names:
        assert hasattr(L, n), n
    assert sorted(hsnf4.EXPORTS) == names


def test_codebook_matches_oracle_bitwise(orc):
    lib_cb = np.array(hsnf4.codebook(), np.float32)
    assert np.array_equal(lib_cb.view(np.uint32), orc.codebook().view(np.uint32))


def test_status_strings():
    L = hsnf4.lib()
    for s in range(7):
        assert L.hsnf4_status_string(s)


def _invalid(rc_call):
    with pytest.raises(hsnf4.HsNf4Error) as e:
        rc_call()
    return e.value


def test_nf4_calls_reject_bad_shapes_before_cuda():
    L = hsnf4.lib()
    fake = 0x10000  # never dereferenced: validation fails first
    rc = L.nf4_quantize_pack(fake, 4, 48, fake, fake, None)
    assert rc == hsnf4.ERR_INVALID and "multiple of 64" in hsnf4.last_error()
    rc = L.nf4_dequant(fake, fake, 0, 64, fake, None)
    assert rc == hsnf4.ERR_INVALID
    rc = L.nf4_quantize_pack(fake + 8, 4, 64, fake, fake, None)
    assert rc == hsnf4.ERR_INVALID and "aligned" in hsnf4.last_error()
    rc = L.nf4_quantize_pack(None, 4, 64, fake, fake, None)
    assert rc == hsnf4.ERR_INVALID and "NULL" in hsnf4.last_error()


def test_lora_calls_validate_rank_shape_workspace():
    import ctypes
    L = hsnf4.lib()
    fake = 0x10000
    W = hsnf4.Nf4WeightC(fake, fake, 128, 256)
    args = lambda r, T, ws: (ctypes.byref(W), fake, T, fake, fake, r, 32.0, fake, fake, fake, ws,
                             None)
    assert L.lora_linear_fwd(*args(4, 64, 1 << 20)) == hsnf4.ERR_INVALID
    assert "rank" in hsnf4.last_error()
    assert L.lora_linear_fwd(*args(16, 0, 1 << 20)) == hsnf4.ERR_INVALID
    need = hsnf4.fwd_workspace_bytes(64, 128, 256, 16)  # upper bound (t_save may be NULL)
    assert L.lora_linear_fwd(*args(16, 64, 1000)) == hsnf4.ERR_OOM
    msg = hsnf4.last_error()
    assert "need" in msg and "1000" in msg  # the detail names needed vs given
    assert need > 64 * 16 * 2
    W2 = hsnf4.Nf4WeightC(fake, fake, 100, 256)
    assert L.lora_linear_fwd(ctypes.byref(W2), fake, 64, fake, fake, 16, 32.0, fake, fake, fake,
                             1 << 20, None) == hsnf4.ERR_INVALID


def test_workspace_sizes():
    assert hsnf4.fwd_workspace_bytes(512, 3584, 3584, 16) >= 512 * 16 * 2 + 512 * 16 * 4
    assert hsnf4.bwd_workspace_bytes(512, 3584, 3584, 16) >= 512 * 16 * 2 + 512 * 16 * 4
    assert hsnf4.fwd_workspace_bytes(100, 64, 64, 8) % 256 == 0


# ---------------------------------------------------------------- slab / ring layout

def _family_desc(fam):
    return hsnf4.layer_desc([(n, k) for _, n, k in synth.FAMILIES[fam].projections()])


def test_layer_layout_is_aligned_and_disjoint(orc):
    d = _family_desc("qwen2.5-7b")
    total = hsnf4.layer_bytes(d)
    assert total % 1024 == 0
    spans = []
    for p, (_, n, k) in enumerate(synth.FAMILIES["qwen2.5-7b"].projections()):
        co, ao = hsnf4.layer_offsets(d, p)
        assert co % 1024 == 0 and ao % 1024 == 0
        spans += [(co, co + n * k // 2), (ao, ao + n * k // 64 * 4)]
    spans.sort()
    assert spans[0][0] == 0 and spans[-1][1] <= total
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    # the payload is the NF4 storage format; alignment adds < 1 KiB per piece
    payload = sum(orc.storage_bytes(n, k) for _, n, k in synth.FAMILIES["qwen2.5-7b"].projections())
    assert payload <= total < payload + 14 * 1024


@pytest.mark.parametrize("bs", [1, 2, 3, 4])
def test_ring_is_two_blocks(bs):
    descs = [_family_desc("llama-3.1-8b")] * 7
    lb = hsnf4.layer_bytes(descs[0])
    assert hsnf4.ring_bytes(descs, bs) == 2 * bs * lb
    assert hsnf4.slab_bytes(descs) == 7 * lb


def test_layout_rejects_bad_descriptors():
    bad = hsnf4.layer_desc([(128, 100)])
    with pytest.raises(hsnf4.HsNf4Error):
        hsnf4.layer_bytes(bad)
    with pytest.raises(hsnf4.HsNf4Error):
        hsnf4.ring_bytes([_family_desc("qwen2.5-7b")], 0)


def test_host_fault_injection_sites():
    hsnf4.inject_fault("copy_enqueue")
    hsnf4.inject_fault(None)
    with pytest.raises(hsnf4.HsNf4Error):
        hsnf4.inject_fault("kernel_trap")


# ---------------------------------------------------------------- dense bf16 base, merge

def test_base_format_validation_before_cuda():
    import ctypes
    L = hsnf4.lib()
    fake = 0x10000
    call = lambda W: L.lora_linear_fwd(ctypes.byref(W), fake, 64, fake, fake, 16, 32.0, fake,
                                       fake, fake, 1 << 20, None)
    # a BF16 base takes absmax = NULL
    assert call(hsnf4.Nf4WeightC(fake, fake, 128, 256, hsnf4.BASE_BF16, 0)) == hsnf4.ERR_INVALID
    assert "absmax = NULL" in hsnf4.last_error()
    # an NF4 base needs absmax
    assert call(hsnf4.Nf4WeightC(fake, None, 128, 256, hsnf4.BASE_NF4, 0)) == hsnf4.ERR_INVALID
    assert "absmax" in hsnf4.last_error()
    # unknown format
    assert call(hsnf4.Nf4WeightC(fake, fake, 128, 256, 7, 0)) == hsnf4.ERR_INVALID
    assert "format" in hsnf4.last_error()
    # one format per group
    Wq = hsnf4.Nf4WeightC(fake, fake, 128, 256, hsnf4.BASE_NF4, 0)
    Wd = hsnf4.Nf4WeightC(fake, None, 128, 256, hsnf4.BASE_BF16, 0)
    arr = (hsnf4.FwdArgs * 2)(hsnf4.FwdArgs(Wq, fake, fake, fake, fake, None),
                              hsnf4.FwdArgs(Wd, fake, fake, fake, fake, None))
    assert L.lora_group_fwd(arr, 2, 64, 16, 32.0, fake, 1 << 30, None) == hsnf4.ERR_INVALID
    assert "one format" in hsnf4.last_error()


def test_merge_validates_before_cuda():
    import ctypes
    L = hsnf4.lib()
    fake = 0x10000
    W = hsnf4.Nf4WeightC(fake, fake, 128, 256, hsnf4.BASE_NF4, 0)
    assert L.lora_merge(ctypes.byref(W), fake, fake, 4, 32.0, fake + 0x1000, None) == \
        hsnf4.ERR_INVALID
    assert "rank" in hsnf4.last_error()
    assert L.lora_merge(ctypes.byref(W), fake, fake, 16, 32.0, fake, None) == hsnf4.ERR_INVALID
    assert "aliases" in hsnf4.last_error()
    assert L.lora_merge(ctypes.byref(W), fake, None, 16, 32.0, fake + 0x1000, None) == \
        hsnf4.ERR_INVALID
    Wbad = hsnf4.Nf4WeightC(fake, fake, 96, 256, hsnf4.BASE_NF4, 0)
    assert L.lora_merge(ctypes.byref(Wbad), fake, fake, 16, 32.0, fake + 0x1000, None) == \
        hsnf4.ERR_INVALID


def test_bf16_layer_layout():
    shapes = [(n, k) for _, n, k in synth.FAMILIES["qwen2.5-7b"].projections()]
    d = hsnf4.layer_desc(shapes, hsnf4.BASE_BF16)
    total = hsnf4.layer_bytes(d)
    spans = []
    for p, (n, k) in enumerate(shapes):
        co, ao = hsnf4.layer_offsets(d, p)
        assert co == ao and co % 1024 == 0
        spans.append((co, co + n * k * 2))
    assert spans[0][0] == 0 and all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    payload = sum(2 * n * k for n, k in shapes)
    assert payload <= total < payload + 7 * 1024
    # 2 B per weight vs 0.5625 B: the pages' 3.56x
    nf4 = hsnf4.layer_bytes(hsnf4.layer_desc(shapes))
    assert abs(total / nf4 - 2 / 0.5625) < 1e-3
    with pytest.raises(hsnf4.HsNf4Error):
        hsnf4.layer_bytes(hsnf4.layer_desc(shapes, 2))


def test_dropout_validation_before_cuda():
    import ctypes
    L = hsnf4.lib()
    fake = 0x10000
    W = hsnf4.Nf4WeightC(fake, fake, 128, 256, hsnf4.BASE_NF4, 0)
    for p in (1.0, -0.25, float("nan")):
        arr = (hsnf4.FwdArgs * 1)(hsnf4.FwdArgs(W, fake, fake, fake, fake, None, p, 0, 1, 2))
        assert L.lora_group_fwd(arr, 1, 64, 16, 32.0, fake, 1 << 30, None) == hsnf4.ERR_INVALID
        assert "dropout_p" in hsnf4.last_error()
        barr = (hsnf4.BwdArgs * 1)(hsnf4.BwdArgs(W, fake, fake, fake, fake, fake, fake, fake, fake,
                                                 p, 0, 1, 2))
        assert L.lora_group_bwd(barr, 1, 64, 16, 32.0, fake, 1 << 30, None) == hsnf4.ERR_INVALID
        assert L.lora_dropout_apply(fake, 64, 256, p, 1, 2, fake, None) == hsnf4.ERR_INVALID
    assert L.lora_dropout_apply(fake, 64, 100, 0.1, 1, 2, fake, None) == hsnf4.ERR_INVALID
    # a forward with dropout needs room for X_d [T, k_in] in its workspace
    plain = hsnf4.FwdArgs(hsnf4.Nf4WeightC(0, 0, 128, 256), 0, 0, 0, 0, 1)
    drop = hsnf4.FwdArgs(hsnf4.Nf4WeightC(0, 0, 128, 256), 0, 0, 0, 0, 1, 0.1, 0, 1, 2)
    assert hsnf4.group_fwd_workspace_bytes([drop], 64, 16) >= \
        hsnf4.group_fwd_workspace_bytes([plain], 64, 16) + 64 * 256 * 2


@pytest.mark.slow
def test_bench_reference_arm_prints_its_json_line():
    """`bench.py --impl reference` (the oracle on the host cores) runs on CPU
    and prints one JSON line with the contract's keys."""
    import json
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--ref-seconds", "0.2"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [l for l in r.stdout.splitlines() if l.startswith("{")][-1]
    d = json.loads(line)
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["config"]["workload"] == "qwen2.5-72b-stack"
    assert d["config"]["layers"] == 80 and "one layer x 80, extrapolated" in d["cpu_baseline"]["sample"]
