"""CPU checks of libtq: it loads, exports every entry point its header
declares, rejects unsupported sizes, and its host-side tables (built in C++
from the same published definitions) agree with the independent oracle."""
import ctypes
import re
from pathlib import Path

import numpy as np
import pytest
import torch

import compressed_decode_attention_quantize_b200 as tq
from oracle import tq_oracle as o

ROOT = Path(__file__).resolve().parent.parent


def _declared_symbols():
    names = set()
    for h in (ROOT / "include").glob("*.h"):
        text = re.sub(r"/\*.*?\*/", "", h.read_text(), flags=re.S)
        names |= set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(tq.library_path())
    declared = _declared_symbols()
    assert "tq_attn_decode" in declared and "tq_quantize" in declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) <= set(tq.EXPORTED) | set(declared)
    assert tq.tq_version().startswith("libtq")


@pytest.mark.parametrize("d,bits_k,bits_v,m,seed", [
    (128, 3, 4, 128, 0), (128, 4, 4, 128, 1), (200, 4, 3, 200, 0), (64, 2, 1, 0, 9),
    (8, 5, 2, 32, 3), (256, 5, 4, 256, 2), (96, 3, 3, 64, 12345678901234), (128, 8, 4, 0, 4),
    (64, 2, 8, 32, 6)])
def test_host_tables_match_oracle(d, bits_k, bits_v, m, seed):
    h = tq.tq_host_tables(d, bits_k, bits_v, m, seed)
    ot = o.make_tables(d, bits_k, bits_v, m, seed)
    assert np.abs(h["Pi"] - ot.Pi).max() < 1e-12
    if m:
        assert np.array_equal(h["S"], ot.S)  # fp16-rounded values agree exactly
    # A 256-level fixed point is ill-conditioned (the Lloyd map contracts by
    # about 1 - 1/L^2 per step), so rounding of 1e-14 in the two sides' cell
    # masses moves it by up to ~1e-10; 16 levels or fewer agree to 1e-12.
    tk = 1e-12 if ot.cb_k.bits <= 4 else 1e-9
    tv = 1e-12 if ot.cb_v.bits <= 4 else 1e-9
    assert np.abs(h["ck"] - ot.cb_k.centroids).max() < tk
    assert np.abs(h["bk"] - ot.cb_k.boundaries).max() < tk
    assert np.abs(h["cv"] - ot.cb_v.centroids).max() < tv
    assert np.abs(h["bv"] - ot.cb_v.boundaries).max() < tv


@pytest.mark.parametrize("args", [(7, 3, 4, 0), (300, 3, 4, 0), (128, 1, 4, 128), (128, 6, 4, 0),
                                  (128, 3, 5, 0), (128, 3, 4, 12), (128, 3, 4, 160), (128, 8, 4, 128),
                                  (128, 3, 7, 0), (128, 9, 4, 0)])
def test_unsupported_sizes_rejected(args):
    with pytest.raises(tq.TQError) as e:
        tq.tq_host_tables(*args, 0)
    assert e.value.status == tq.TQ_ERR_UNSUPPORTED
    with pytest.raises(tq.TQError):
        tq.tq_init(*args, 0)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_init_without_device_reports_cuda_error():
    with pytest.raises(tq.TQError) as e:
        tq.tq_init(128, 3, 4, 128, 0)
    assert "cuda" in str(e.value).lower()


def test_norm_correction_flags_validated_before_any_device_call():
    with pytest.raises(tq.TQError) as e:
        tq.tq_init_ex(128, 3, 4, 128, 0, tq.TQ_NC_KEYS)   # keys with QJL
    assert "norm correction" in str(e.value)
    with pytest.raises(tq.TQError) as e:
        tq.tq_init_ex(128, 3, 4, 0, 0, 8)
    assert "flag" in str(e.value)
    with pytest.raises(tq.TQError) as e:
        tq.tq_init_ex(128, 3, 4, 128, 0, tq.TQ_NORM_F16)   # binary16 norms with QJL keys
    assert "fp16 norms" in str(e.value)
    with pytest.raises(ValueError):
        tq.Context.variant("k2v2", 128)
    assert set(tq.VARIANTS) == {"k3v4", "k4v4", "k3v4_nc", "4bit_nc", "3bit_nc", "k8v4"}
