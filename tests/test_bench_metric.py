"""The bench's work counts on CPU.  The metric's FLOPs are 4*d*r_i*c_j summed
over the kept (query block i, key block j) pairs, r_i and c_j the valid
tokens of the blocks (the last block of a sequence may be short), and the
mask's algorithmic bytes are Q and K read once plus the CSR written.  Both
are checked against a brute-force sum over random CSR masks laid out the way
the library writes them (ascending rows with gaps between them).  The
reference arm (the oracle on the host's cores) is run once on the small
workload for its JSON line."""
from dataclasses import replace
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import bench
from image_dits_b200.workload import WORKLOADS


def _random_mask(wl, rng):
    """A CSR mask over all B*H*T_b rows: each row keeps a random ascending
    subset of the T_b key blocks (the last block in about half of the rows,
    and some rows keep every block), stored at offsets with gaps."""
    Tb = wl.num_blocks
    rows = wl.batch * wl.heads * Tb
    starts, counts, cols = [], [], []
    pos = 0
    dense = np.zeros((rows, Tb), dtype=bool)
    for r in range(rows):
        if r % 7 == 3:
            kept = np.arange(Tb)
        else:
            n = int(rng.integers(1, Tb + 1))
            kept = np.sort(rng.choice(Tb, size=n, replace=False))
        dense[r, kept] = True
        pos += int(rng.integers(0, 3))              # a gap before the row
        starts.append(pos)
        counts.append(len(kept))
        cols.extend(int(j) for j in kept)
        pos += len(kept)
    col_idx = np.full(pos + 2, -7, dtype=np.int32)   # gaps hold garbage
    at = 0
    for s, c in zip(starts, counts):
        col_idx[s:s + c] = cols[at:at + c]
        at += c
    mask = SimpleNamespace(row_start=torch.tensor(starts, dtype=torch.int32),
                           row_count=torch.tensor(counts, dtype=torch.int32),
                           col_idx=torch.from_numpy(col_idx))
    mask.kept_pairs = lambda: int(sum(counts))
    return mask, dense


def _brute_flops(wl, dense):
    Tb, N, d = wl.num_blocks, wl.num_tokens, wl.head_dim
    valid = np.array([min(64, N - 64 * b) for b in range(Tb)], dtype=np.int64)
    rows_i = np.tile(valid, dense.shape[0] // Tb)     # row r is query block r mod T_b
    total = 0
    for r in range(dense.shape[0]):
        total += 4 * d * int(rows_i[r]) * int(valid[dense[r]].sum())
    return float(total)


@pytest.mark.parametrize("wl", [
    WORKLOADS["tiny"],                                                    # N a multiple of 64
    replace(WORKLOADS["tiny"], name="ragged", frames=3, height=7, width=9),  # last block of 61 tokens
    replace(WORKLOADS["tiny"], name="text", text_tokens=37),             # N = 1024 + 37
    replace(WORKLOADS["tiny"], name="short", frames=1, height=5, width=7, heads=3),  # one block of 35
])
def test_kept_flops_match_brute_force(wl):
    rng = np.random.default_rng(5)
    mask, dense = _random_mask(wl, rng)
    assert bench.kept_flops_from_mask(mask, wl) == _brute_flops(wl, dense)


def test_kept_flops_of_a_full_mask_is_dense_attention():
    """keep = 1: every pair is kept, so the count is dense attention's 4*d*N^2
    per head (closed form)."""
    wl = replace(WORKLOADS["tiny"], name="ragged", frames=3, height=7, width=9)
    Tb = wl.num_blocks
    rows = wl.batch * wl.heads * Tb
    mask = SimpleNamespace(row_start=torch.arange(rows, dtype=torch.int32) * Tb,
                           row_count=torch.full((rows,), Tb, dtype=torch.int32),
                           col_idx=torch.arange(Tb, dtype=torch.int32).repeat(rows))
    expect = 4.0 * wl.head_dim * wl.num_tokens ** 2 * wl.batch * wl.heads
    assert bench.kept_flops_from_mask(mask, wl) == expect


def test_mask_bytes():
    wl = WORKLOADS["tiny"]
    mask, _ = _random_mask(wl, np.random.default_rng(1))
    qk = 2 * wl.batch * wl.heads * wl.num_tokens * wl.head_dim * 2
    csr = 4 * (2 * mask.row_count.numel() + mask.kept_pairs())
    assert bench.mask_bytes(wl, mask) == float(qk + csr)


def test_attention_traffic_figure_covers_the_compulsory_bytes():
    """The measured DRAM bytes per token-head of the attention kernel are at
    least its compulsory traffic (Q, K, V read once and O written once in bf16
    at d = 128: 1,024 bytes) and not far above it (K/V re-reads hit L2)."""
    assert 1024 <= bench.ATTN_DRAM_BYTES_PER_TOKEN_HEAD <= 1.2 * 1024
    assert len(bench.ATTN_TRAFFIC_BUILD) >= 7


def test_reference_arm_line():
    """`bench.py --impl reference` (the oracle on the host's cores, the arm the
    driver times beside the library) runs without a GPU and prints one JSON
    line with the contract's keys."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "TFLOP/s"
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] >= 3 and d["n_gpus"] == 1
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_under_torchrun():
    """Launched as the driver launches N > 1 (torchrun, two processes): rank 0
    alone runs the oracle and prints the one line; the other rank exits 0
    without work."""
    import json
    import os
    import socket
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                        "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(root, "bench.py"),
                        "--impl", "reference", "--gpus", "2", "--workload", "tiny", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
