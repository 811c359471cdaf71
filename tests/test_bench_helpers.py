"""Host-side helpers of the benchmark and of sequence sharding (CPU)."""
import json
import os

import numpy as np
import torch

import bench
from linear_attention_linattn_b200 import seqshard

SRC = """// a kernel
int f(int x) {  /* the body */
  return x + 1;  // one more
}
"""


def test_code_hash_ignores_comments_but_not_code(tmp_path):
    a, b, c = tmp_path / "a.cu", tmp_path / "b.cu", tmp_path / "c.cu"
    a.write_text(SRC)
    b.write_text(SRC.replace("// a kernel", "// the same kernel, reworded\n\n"))
    c.write_text(SRC.replace("x + 1", "x + 2"))
    assert bench.code_hash(str(a)) == bench.code_hash(str(b))
    assert bench.code_hash(str(a)) != bench.code_hash(str(c))


def test_kernel_traffic_needs_the_captured_code(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text(SRC)
    (tmp_path / "profiles").mkdir()
    rec = {"K3 | w": {"dram_bytes_per_launch": 123, "source": "k.cu",
                      "source_code_sha256": bench.code_hash(str(src))}}
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_traffic("K3", "w") == 123.0
    assert bench.kernel_traffic("K1", "w") is None          # no record
    src.write_text(SRC + "// a comment only\n")
    assert bench.kernel_traffic("K3", "w") == 123.0         # comments do not count
    src.write_text(SRC.replace("x + 1", "x - 1"))
    assert bench.kernel_traffic("K3", "w") is None          # the code changed


def test_committed_traffic_record_matches_the_kernel_source():
    """The record the benchmark reports was taken on the code of the kernel as committed."""
    with open(os.path.join(bench.ROOT, "profiles", "ncu_traffic.json")) as f:
        table = json.load(f)
    for key, rec in table.items():
        path = os.path.join(bench.ROOT, rec["source"])
        assert bench.code_hash(path) == rec["source_code_sha256"], key


def test_pack_state_layout():
    B, H, d = 2, 3, 4
    S = torch.arange(B * H * d * d, dtype=torch.float32).reshape(B, H, d, d)
    z = -torch.arange(B * H * d, dtype=torch.float32).reshape(B, H, d)
    p = seqshard.pack_state(S, z)
    assert p.shape == (B, H, d * d + d) and p.is_contiguous()
    assert np.array_equal(p[..., :d * d].numpy(), S.reshape(B, H, -1).numpy())
    assert np.array_equal(p[..., d * d:].numpy(), z.numpy())
