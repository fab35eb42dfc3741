"""Host-side helpers of bench.py (CPU): the kept-work count behind TFLOP/s on
kept blocks, the all-blocks CSR used for the entropy-overhead reference, and
the rule that the recorded DRAM traffic is reported only for the kernel
source it was measured on."""
import json
import os

import numpy as np

import bench
from entropy_adaptive_radius_b200 import inputs, workloads
from oracle import tra_oracle as O


def test_kept_pair_tokens_counts_tail_blocks_exactly():
    # N = 300 with 128-blocks: sizes 128, 128, 44
    heads, N, B = 2, 300, 128
    m = np.array([[[1, 0, 1], [0, 1, 0], [1, 1, 1]],
                  [[0, 0, 1], [1, 0, 0], [0, 0, 0]]], bool)
    rp, ci = inputs.csr_from_block_mask(m)
    sz = [128, 128, 44]
    expect = sum(sz[q] * sz[k] for h in range(heads) for q in range(3) for k in range(3) if m[h, q, k])
    assert bench.kept_pair_tokens(rp.ravel(), ci, heads, N, B, B) == expect
    # against the token-level key mask of the oracle
    km = [O.key_mask_from_blocks(m[h], np.arange(N), B, B, N).sum() for h in range(heads)]
    assert expect == sum(km)


def test_executed_over_kept_counts_the_union_of_two_query_blocks():
    """64-token query blocks pair up in 128-row tiles that run the union of
    their two key-block lists for all 128 rows."""
    N, B = 256 + 40, 64           # blocks of 64, 64, 64, 64, 40
    m = np.zeros((1, 5, 5), bool)
    m[0, 0, 0] = m[0, 1, 1] = True                  # disjoint: union of 2 for 128 rows
    m[0, 2, [2, 3]] = m[0, 3, [2, 3]] = True        # identical lists: no extra work
    m[0, 4, [0, 4]] = True                          # last tile holds one 40-row block
    rp, ci = inputs.csr_from_block_mask(m)
    kept = 64 * 64 * 2 + 64 * 128 * 2 + 40 * (64 + 40)
    executed = 128 * 128 + 128 * 128 + 40 * (64 + 40)
    got = bench.executed_over_kept(rp.ravel(), ci, 1, N, B, B)
    assert abs(got - executed / kept) < 1e-12
    assert bench.executed_over_kept(rp.ravel(), ci, 1, N, 128, 128) == 1.0


def test_full_csr_keeps_every_block():
    heads, N, B = 3, 1000, 128
    rp, ci = bench.full_csr(heads, N, B, "cpu")
    nqb = -(-N // B)
    rp = rp.numpy().reshape(heads, nqb + 1)
    ci = ci.numpy()
    assert rp[0, 0] == 0 and rp[-1, -1] == heads * nqb * nqb
    for h in range(heads):
        for q in range(nqb):
            assert np.array_equal(ci[rp[h, q]:rp[h, q + 1]], np.arange(nqb))


def test_measured_traffic_needs_the_captured_source(tmp_path, monkeypatch):
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "dram_traffic_wan14b.txt")))
    wl = workloads.WAN14B
    got = bench.measured_traffic(wl, "dense_attn_entropy")
    src = open(os.path.join(bench.ROOT, rec["source"]), "rb").read()
    if bench.code_sha256(os.path.join(bench.ROOT, rec["source"])) == rec["source_code_sha256"]:
        assert got == rec["dense_attn_entropy"]["traffic_bytes"]
    else:
        assert got is None
    # another workload, or changed code, gives no figure
    assert bench.measured_traffic(workloads.WAN13B, "dense_attn_entropy") is None
    fake = dict(rec, source_code_sha256="0" * 64)
    p = tmp_path / "profiles"
    p.mkdir()
    (p / "dram_traffic_wan14b.txt").write_text(json.dumps(fake))
    (tmp_path / os.path.dirname(rec["source"])).mkdir(parents=True)
    (tmp_path / rec["source"]).write_bytes(src)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic(wl, "dense_attn_entropy") is None


def test_traffic_record_is_near_the_algorithmic_bytes():
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "dram_traffic_wan14b.txt")))
    wl = workloads.WAN14B
    alg = 4 * wl.heads * wl.N * wl.d * 2 + 4 * wl.heads * wl.N
    assert rec["dense_attn_entropy"]["algorithmic_bytes"] == alg
    for k in ("dense_attn_entropy", "block_sparse_attn"):
        r = rec[k]
        assert r["traffic_bytes"] == r["dram_read_bytes"] + r["dram_write_bytes"]
        assert 0.95 < r["traffic_bytes"] / r["algorithmic_bytes"] < 1.1


def test_code_hash_ignores_comments_only(tmp_path):
    a = tmp_path / "a.cu"
    b = tmp_path / "b.cu"
    c = tmp_path / "c.cu"
    a.write_text("int f(int x) {  // twice\n  return 2 * x; }\n")
    b.write_text("/* doubles */\nint f(int x) {\n  return 2 * x;\n}\n")
    c.write_text("int f(int x) { return 3 * x; }\n")
    assert bench.code_sha256(str(a)) == bench.code_sha256(str(b))
    assert bench.code_sha256(str(a)) != bench.code_sha256(str(c))
