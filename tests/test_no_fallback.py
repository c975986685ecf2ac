"""The product path has no CPU fallback: without a GPU every compute call refuses CPU tensors,
and without the built library the binding does not import."""
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def mla():
    from deepseek_mla_latent_b200 import build
    build.build()
    from deepseek_mla_latent_b200 import mla as m
    return m


def test_compute_calls_refuse_host_tensors(mla):
    from deepseek_mla_latent_b200 import workloads as wl
    d = mla.dims_from(wl.V3)
    bf = torch.bfloat16
    q = torch.zeros(2, 128, 192, dtype=bf)
    wkv_b = torch.zeros(128 * 256, 512, dtype=bf)
    q_abs = torch.zeros(2, 128, 512, dtype=bf)
    kv, pe = torch.zeros(256, 512, dtype=bf), torch.zeros(256, 64, dtype=bf)
    cu = torch.tensor([0, 128, 256], dtype=torch.int32)
    calls = [
        lambda: mla.absorb_q(d, q, wkv_b),
        lambda: mla.attn_decode(d, q_abs, q, kv, pe, cu, 128),
        lambda: mla.attn_decode_out(d, q_abs, q, kv, pe, cu, 128, wkv_b),
        lambda: mla.attn_paged(d, q_abs, q, torch.tensor([128, 128], dtype=torch.int32), 128, kv, pe,
                               torch.tensor([[0, 1], [2, 3]], dtype=torch.int32), 64),
        lambda: mla.out_proj(d, q_abs, wkv_b),
        lambda: mla.expand_kv(d, kv, wkv_b, 1, 256),
        lambda: mla.append_latent(d, kv[:4], pe[:4], torch.zeros(4, dtype=torch.int32),
                                  torch.arange(4, dtype=torch.int64), kv, pe),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="CUDA tensor"):
            call()


def test_binding_needs_the_library(tmp_path):
    """Loading from a path where the library is missing raises ImportError (no fallback)."""
    code = ("import sys; sys.path.insert(0, %r)\n"
            "from deepseek_mla_latent_b200 import _lib\n"
            "try:\n    _lib.load_library(%r)\nexcept ImportError as e:\n    print('ImportError', e)\n"
            % (ROOT, str(tmp_path / "missing.so")))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120)
    assert "ImportError" in r.stdout, r.stdout + r.stderr
