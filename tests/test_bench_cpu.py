"""bench.py on the host: its reference arm (the oracle timed on the CPU) runs
and prints one well-formed JSON line, and every global name its functions use
is defined (a broken bench must fail here, not on the GPU machine)."""
import builtins
import dis
import importlib.util
import json
import os
import subprocess
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _loaded_globals(code):
    """Names the code (and every function or lambda nested in it) loads as globals."""
    names = {ins.argval for ins in dis.get_instructions(code) if ins.opname == "LOAD_GLOBAL"}
    for c in code.co_consts:
        if isinstance(c, types.CodeType):
            names |= _loaded_globals(c)
    return names


def test_bench_functions_load_only_defined_globals():
    b = _load_bench()
    for name, obj in vars(b).items():
        if isinstance(obj, types.FunctionType) and obj.__module__ == b.__name__:
            undefined = sorted(n for n in _loaded_globals(obj.__code__)
                               if n not in vars(b) and not hasattr(builtins, n))
            assert not undefined, (name, undefined)
    for fn in ("main", "run_ours", "run_reference", "run_e2e_pipelined"):
        assert callable(getattr(b, fn, None)), fn


def test_reference_arm_prints_its_json_line():
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1", "--warmup", "0",
         "--ref-seconds", "0.05"],
        cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    line = [l for l in out.stdout.splitlines() if l.startswith("{")][-1]
    rec = json.loads(line)
    assert rec["impl"] == "reference"
    assert rec["value"] > 0 and rec["steps"] == 1 and rec["warmup"] == 0
    assert rec["config"]["workload"] == "dsv3_b64_h128_t4096_paged"
    # the same config dict as the GPU arm prints for this workload
    import mla_workloads as mw
    b = _load_bench()
    assert rec["config"] == json.loads(json.dumps(b.config_dict(mw.make_config(2, seed=0), 1)))
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] >= 1
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["e2e"]["d2h_bytes_per_step"] == 0
    assert rec["higher_is_better"] is True


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_reference_arm_under_torchrun_two_ranks():
    # two ranks on gloo: rank 0 alone times the oracle and prints the line,
    # rank 1 exits without work; both exit 0
    out = subprocess.run(
        [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
         "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
         os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
         "--ref-seconds", "0.05"],
        cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0


def _ranks_body(rank, port, results):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE="2", RANK=str(rank),
                      LOCAL_RANK=str(rank))
    b = _load_bench()
    world, r, _ = b.dist_setup(2)
    try:
        b.barrier(world)
        results[r] = b.max_over_ranks(float(10 * r + 1), world)
    finally:
        dist.destroy_process_group()


def test_barrier_and_max_over_ranks_on_gloo():
    import torch.multiprocessing as mp
    port = _free_port()
    with mp.Manager() as m:
        results = m.dict()
        ctx = mp.get_context("spawn")
        ps = [ctx.Process(target=_ranks_body, args=(r, port, results)) for r in range(2)]
        for p in ps:
            p.start()
        for p in ps:
            p.join(300)
        assert all(p.exitcode == 0 for p in ps)
        assert dict(results) == {0: 11.0, 1: 11.0}
