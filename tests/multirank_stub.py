"""One rank of bench.py's multi-rank run with the GPU step replaced by a
stand-in (test infrastructure; run by tests/test_multirank.py through
bench.spawn_ranks, i.e. torch.distributed.run with gloo ranks on the CPU).

The stand-in keeps the workload accounting of the real step (visible pairs,
useful FLOPs, tokens) and reports fixed per-rank times: rank r takes
(2 + r) ms per step, so the job's step time is the slowest rank's."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from block_sparse_attention_kunlun_b200 import flops as F  # noqa: E402


class StubRunner:
    def __init__(self, ba, w, inp, dev, rope=False, gdpa=None, mx=False):
        self.w, self.inp = w, inp
        self.lens = inp["lengths"].numpy()
        self.skip_np = inp["skip"].numpy() if inp["skip"] is not None else None
        self.T, self.H, self.D = inp["q"].shape
        self.pairs = F.visible_pairs(self.lens, w.block, w.window, self.skip_np)
        self.flops = F.step_flops(self.pairs, self.H, self.D)
        self.bytes = F.step_bytes(self.T, self.H, self.D)
        self.launches_per_step = 5
        self.rank = int(os.environ["RANK"])
        self.fused = False  # the two-pass backward's kernel accounting
        self.kernel_names = dict(bench.KERNEL_NAMES)

    def timed(self, K, warmup, barrier, clocks=None):
        barrier()
        ms = 2.0 + self.rank
        return ms * K, {"fwd": ms / 4, "bwd_dq": ms / 4, "bwd_dkdv": ms / 2}

    def kernel_stats(self, ms_k):
        return bench.Runner.kernel_stats(self, ms_k)


if __name__ == "__main__":
    bench.main(runner_cls=StubRunner)
