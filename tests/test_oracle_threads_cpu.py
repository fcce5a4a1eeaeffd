"""The oracle's results do not depend on its OpenMP thread count (every output is computed by one
thread in a fixed order), so the CPU baseline and the parity references agree on any host."""
import os
import subprocess
import sys

import numpy as np

from block_sparse_attention_blocks_b200.workloads import f32_to_bf16_bits

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_oracle_results_do_not_depend_on_the_thread_count(orc, tmp_path):
    # every output is computed by one thread in a fixed order: one thread and many agree bit for bit
    rng = np.random.default_rng(36)
    BH, N, d, bs = 3, 200, 16, 32
    q, k, v = (f32_to_bf16_bits(rng.standard_normal((BH, N, d)).astype(np.float32)) for _ in range(3))
    np.savez(tmp_path / "in.npz", q=q, k=k, v=v)
    code = (
        "import numpy as np, oracle as o\n"
        f"z = np.load(r'{tmp_path / 'in.npz'}')\n"
        "qp, kp = o.pool_blocks(z['q'], 32), o.pool_blocks(z['k'], 32)\n"
        "s = o.select(qp, kp, 2, 0.8, 0.25)\n"
        "out = o.masked_attention(z['q'], z['k'], z['v'], s.mask, 32, 0.25)\n"
        f"np.savez(r'{tmp_path / 'out1.npz'}', qp=qp, mask=s.mask, out=out)\n")
    env = dict(os.environ, OMP_NUM_THREADS="1")
    subprocess.run([sys.executable, "-c", code], check=True, env=env, cwd=ROOT)
    one = np.load(tmp_path / "out1.npz")
    qp, kp = orc.pool_blocks(q, bs), orc.pool_blocks(k, bs)
    s = orc.select(qp, kp, 2, 0.8, 0.25)
    out = orc.masked_attention(q, k, v, s.mask, bs, 0.25)
    assert np.array_equal(one["qp"], qp) and np.array_equal(one["mask"], s.mask)
    assert np.array_equal(one["out"], out)
