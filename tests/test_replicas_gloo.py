"""The multi-GPU path is replicas only: each rank runs its own model and the
ranks exchange nothing but the step time. These tests run that host logic as
two gloo ranks on the CPU (rendezvous on 127.0.0.1): the max-over-ranks step
time, the whole-job throughput, and the reference arm's non-zero ranks
exiting without work, and the reference arm's JSON line."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.join(os.path.dirname(os.path.abspath(__file__)), '..')

WORKER = r'''
import datetime, json, os, sys
sys.path.insert(0, os.environ["REPO_ROOT"])
import torch.distributed as dist
import bench
ws, rank, local = bench._dist()
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
try:
    bench._barrier(ws)
    value, ms = bench.replica_throughput(2048, 10.0 + rank, ws)
    mx = bench._max_over_ranks(3.0 * rank, ws)
    print(json.dumps({"rank": rank, "ws": ws, "value": value, "ms": ms, "max": mx}), flush=True)
finally:
    dist.destroy_process_group()
'''


def _free_port() -> int:
    s = socket.socket()
    s.bind(('127.0.0.1', 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _env(rank: int, ws: int, port: int) -> dict:
    env = dict(os.environ)
    env.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(ws), MASTER_ADDR='127.0.0.1',
               MASTER_PORT=str(port), REPO_ROOT=ROOT)
    return env


def test_two_replicas_aggregate_over_gloo():
    port = _free_port()
    procs = [subprocess.Popen([sys.executable, '-c', WORKER], env=_env(r, 2, port), stdout=subprocess.PIPE,
                              stderr=subprocess.PIPE, text=True) for r in range(2)]
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=180)
        assert p.returncode == 0, err
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o['ws'] == 2
        assert o['ms'] == 11.0                        # the slower rank's time
        assert abs(o['value'] - 2 * 2048 / 0.011) < 1e-6
        assert o['max'] == 3.0
    assert sorted(o['rank'] for o in outs) == [0, 1]


def test_reference_arm_other_ranks_exit_without_work():
    r = subprocess.run([sys.executable, os.path.join(ROOT, 'bench.py'), '--impl', 'reference', '--gpus', '2',
                        '--steps', '1', '--warmup', '0'], env=_env(1, 2, _free_port()), capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ''


def test_reference_arm_prints_the_contract_line():
    """Rank 0 of the reference arm times the CPU oracle on a bounded sample and
    prints one JSON line with the same metric and workload as the GPU arm."""
    sys.path.insert(0, ROOT)
    import bench
    r = subprocess.run([sys.executable, os.path.join(ROOT, 'bench.py'), '--impl', 'reference', '--steps', '1',
                        '--warmup', '0'], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith('{')]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ('metric', 'value', 'unit', 'n_gpus', 'steps', 'warmup', 'ms_per_step', 'higher_is_better',
                'scaling', 'vs_baseline', 'dtype', 'data', 'config', 'cpu_baseline', 'e2e'):
        assert key in d, key
    assert d['impl'] == 'reference' and d['metric'] == bench.METRIC and d['unit'] == 'tokens/s'
    assert d['value'] > 0 and d['higher_is_better'] is True and d['steps'] == 1
    import argparse
    assert d['config'] == bench.workload_config(1, argparse.Namespace(paged=False))
    cb = d['cpu_baseline']
    assert cb['kind'] == 'oracle' and cb['value'] == d['value'] and cb['cores'] >= 1 and cb['sample']
    assert d['e2e'] == {'value': d['value'], 'unit': 'tokens/s', 'h2d_bytes_per_step': 0, 'd2h_bytes_per_step': 0}
