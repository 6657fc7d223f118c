"""Multi-rank host logic of bench.py on CPU: two gloo ranks, the barrier, and
the max-over-ranks step time that `value` divides by.  The data path has no
collective (token-parallel replicas), so this is all N>1 adds."""
import os
import socket
import subprocess
import sys
import textwrap

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


CHILD = textwrap.dedent("""
    import os, sys
    sys.path.insert(0, {root!r})
    import bench
    d = bench.Dist(2)
    d.barrier()
    local = 10.0 + d.rank            # rank 1 is the slower one
    m = d.max(local)
    assert m == 11.0, m
    d.barrier()
    print(f"rank {{d.rank}} ok {{m}}")
    d.close()
""")


def test_two_rank_gloo_max_and_barrier(tmp_path):
    port = _free_port()
    script = tmp_path / "child.py"
    script.write_text(CHILD.format(root=ROOT))
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.STDOUT, text=True))
    outs = [p.communicate(timeout=120)[0] for p in procs]
    for r, (p, o) in enumerate(zip(procs, outs)):
        assert p.returncode == 0, o
        assert f"rank {r} ok 11.0" in o


def test_world_size_mismatch_is_rejected():
    import pytest

    import bench
    with pytest.raises(SystemExit):
        bench.Dist(2)   # WORLD_SIZE unset -> 1
