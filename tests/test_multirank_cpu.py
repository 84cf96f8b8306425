"""The multi-rank paths of the benchmark on CPU (gloo, two ranks).

The operator shards over images with no exchange, so N GPUs run N replicas;
the only cross-rank step is the max-over-ranks reduction of the timings,
tested here with gloo, plus the reference arm, which rank 0 alone runs."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

from tests.conftest import ROOT


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        mine = [1.0 + rank, 10.0 - rank, 3.0]
        results[rank] = bench.max_over_ranks(mine, "cpu")
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        results = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, port, results)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        assert results[0] == results[1] == [2.0, 10.0, 3.0]


def test_bench_reference_arm_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600,
                         env={**os.environ, "OMP_NUM_THREADS": "1"})
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    # the reference arm's config is the GPU arm's, key for key (the sample note
    # lives in cpu_baseline)
    sys.path.insert(0, ROOT)
    import bench
    import gen
    wl = gen.WORKLOADS[bench.DEFAULT_WORKLOAD]
    assert d["config"] == bench.workload_config(wl, wl.backward or wl.dtype == "f32", 2)
    assert "sample" not in d["config"] and "sample" in d["cpu_baseline"]


def test_bench_module_resolves_every_name():
    """Every name a function of bench.py reads at module level is defined
    (the GPU-only legs of the benchmark cannot run here, so this catches a
    helper lost in an edit before a GPU run does)."""
    import ast
    import builtins
    import importlib.util

    path = os.path.join(ROOT, "bench.py")
    spec = importlib.util.spec_from_file_location("bench_static_check", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    tree = ast.parse(open(path).read())
    missing = set()
    # module-level functions and class methods; a nested function is checked as
    # part of the function around it (its free names are that function's locals)
    tops = [n for n in tree.body if isinstance(n, ast.FunctionDef)]
    tops += [m for c in tree.body if isinstance(c, ast.ClassDef) for m in c.body
             if isinstance(m, ast.FunctionDef)]
    for fn in tops:
        local = {a.arg for a in fn.args.args + fn.args.kwonlyargs}
        if fn.args.vararg:
            local.add(fn.args.vararg.arg)
        for n in ast.walk(fn):
            if isinstance(n, ast.Name) and isinstance(n.ctx, ast.Store):
                local.add(n.id)
            elif isinstance(n, (ast.FunctionDef, ast.Lambda)) and n is not fn:
                if isinstance(n, ast.FunctionDef):
                    local.add(n.name)
                local.update(a.arg for a in n.args.args)
            elif isinstance(n, (ast.Import, ast.ImportFrom)):
                local.update((a.asname or a.name).split(".")[0] for a in n.names)
            elif isinstance(n, ast.comprehension):
                for t in ast.walk(n.target):
                    if isinstance(t, ast.Name):
                        local.add(t.id)
            elif isinstance(n, ast.ExceptHandler) and n.name:
                local.add(n.name)
            elif isinstance(n, (ast.With, ast.AsyncWith)):
                for it in n.items:
                    if it.optional_vars is not None:
                        for t in ast.walk(it.optional_vars):
                            if isinstance(t, ast.Name):
                                local.add(t.id)
        for n in ast.walk(fn):
            if (isinstance(n, ast.Name) and isinstance(n.ctx, ast.Load) and n.id not in local
                    and not hasattr(mod, n.id) and not hasattr(builtins, n.id)):
                missing.add((fn.name, n.id))
    assert not missing, sorted(missing)



def test_bench_config_names_the_deterministic_backward():
    """`--deterministic` changes what the step's backward is, so the config
    object (the same for both arms) says so; without it the config is the
    default one."""
    sys.path.insert(0, ROOT)
    import bench
    import gen
    wl = gen.WORKLOADS["internimage_l_stage2_bwd_bf16_n32_48x48_c320"]
    plain = bench.workload_config(wl, True, 1)
    det = bench.workload_config(wl, True, 1, True)
    assert "deterministic" not in plain["workload"] and "deterministic" in det["workload"]
    assert {k: v for k, v in det.items() if k != "workload"} == \
        {k: v for k, v in plain.items() if k != "workload"}
    ap_src = open(os.path.join(ROOT, "bench.py")).read()
    assert '"--deterministic"' in ap_src
