"""Host-side logic of bench.py's multi-GPU (replica) mode, on CPU.

bench.py --gpus N runs N independent replicas (the single-layer product has no data-path
collective) and reports the slowest rank's time: two gloo ranks on CPU check that every
rank gets the maximum. The batch-chunk schedule behind the launch count is checked
against its definition.
"""

import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

import importlib.util  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = _bench()
        mine = 1.5 + rank * 2.25  # per-rank timings differ
        out[rank] = b.max_over_ranks(mine, dist, "cpu")
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        ctx = mp.get_context("spawn")
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        assert out[0] == out[1] == pytest.approx(1.5 + 2.25)


def test_max_without_process_group_is_identity():
    assert _bench().max_over_ranks(3.25, None, "cpu") == 3.25


def test_decoder_stream_matrices():
    # the decoder7b workload streams, per layer, the seven Llama-7B matrix shapes in layer
    # order with two bases and a rank-256 correction each (1,714,176,000 algorithmic bytes
    # per 32-layer stream at M=1, the figure the workload table gives)
    b = _bench()
    mats = b.base_matrices("decoder7b", 1)
    assert [(L.out, L.in_) for (L, _) in mats] == [(4096, 4096)] * 4 + [(11008, 4096)] * 2 + [(4096, 11008)]
    assert all(L.K == 2 and L.rank == 256 and L.n_sal == 0 for (L, _) in mats)
    total = sum(b.algorithmic_bytes(L, 1, 2, 2) for (L, _) in mats) * b.DECODER_LAYERS
    assert total == 1_714_176_000


def test_fluxbin_workloads_and_their_bytes():
    # FluxBin 2b-g128 and 2b-s16-g128 on 4096 x 4096 ("FluxBin", Sec. 4 configurations):
    # grouped row scales of 128 columns; 16 salient columns in each of the 32 groups for the
    # refined one. The bench's byte accounting (restated so that the bench does not import
    # the oracle) agrees with the oracle's.
    import oracle
    b = _bench()
    (Lg, Xg), = b.base_matrices("fluxbin4096_g128", 1)
    (Ls, Xs), = b.base_matrices("fluxbin4096_s16", 8)
    assert Lg.group == Ls.group == 128 and Lg.K == Ls.K == 2 and getattr(Lg, "ref_K", 0) == 0
    assert Ls.ref_K == 2 and len(Ls.ref_idx) == 512 and Xs.shape == (8, 4096)
    assert all(((Ls.ref_idx >= 128 * j) & (Ls.ref_idx < 128 * (j + 1))).sum() == 16 for j in range(32))
    for L, M in ((Lg, 1), (Ls, 1), (Ls, 8)):
        assert b.algorithmic_bytes(L, M, 2, 2) == oracle.algorithmic_bytes(L, M, "bf16", "bf16")
    assert b.algorithmic_bytes(Ls, 1, 2, 2) - b.algorithmic_bytes(Lg, 1, 2, 2) == 1_052_672


def test_traffic_record_sums_the_refinement_launch_and_checks_the_sources(tmp_path):
    # roofline.traffic is the DRAM bytes of one GEMV from committed captures: the dominant
    # launch plus, for a refined layer, its refinement launch; null when either capture was
    # taken from other kernel sources
    import json
    b = _bench()
    dig = b.sources_digest()
    rec = {"fluxbin4096_s16_M1": {"sources": dig, "dram_bytes_per_launch": 4_800_000},
           "fluxbin4096_s16_M1_refine": {"sources": dig, "dram_bytes_per_launch": 1_100_000},
           "attn4096_M1": {"sources": dig, "dram_bytes_per_launch": 4_276_000},
           "attn4096_M2": {"sources": "0000000000000000", "dram_bytes_per_launch": 4_300_000},
           "lowrank5120_M1": {"sources": dig, "dram_bytes_per_launch": 7_300_000},
           "lowrank5120_M1_refine": {"sources": "0000000000000000", "dram_bytes_per_launch": 1}}
    f = tmp_path / "traffic.json"
    f.write_text(json.dumps(rec))
    b.TRAFFIC_FILE = str(f)
    assert b.traffic_for("fluxbin4096_s16", 1) == 5_900_000
    assert b.traffic_for("attn4096", 1) == 4_276_000
    assert b.traffic_for("attn4096", 2) is None        # captured from other sources
    assert b.traffic_for("lowrank5120", 1) is None     # its second launch was
    assert b.traffic_for("fluxbin4096_g128", 1) is None  # never captured


def test_reference_arm_prints_one_contract_line():
    # bench.py --impl reference times the oracle on the host cores (no GPU needed) and
    # prints one JSON line with the base contract's keys, the same metric and config as
    # the CUDA arm, and an e2e entry that moves no bytes across PCIe.
    import json
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "1"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["metric"] == "M=1 binary-GEMV effective HBM GB/s" and d["unit"] == "GB/s"
    assert d["config"]["workload"].startswith("attn4096") and d["config"]["M"] == 1
    assert d["steps"] == 1 and d["warmup"] == 1 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["unit"] == d["unit"]
