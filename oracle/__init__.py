"""fp64 CPU oracle of the timestep-forced streaming denoising step.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference leg may import or run anything in this
package.  The CUDA path in ``streaming_causal_video_timestep_b200`` shares no
code with it: neither imports the other; both take their inputs from the
seeded generators in ``workloads``.

What it computes (Live Avatar, arXiv 2512.04677, as described on the pages):
  * block-causal attention of a 3-latent-frame block over [sink | rolling
    window | itself] (10100.com article, training-framework figure caption:
    "block-independent noise + causal mask"; papernotes note, 整体框架);
  * a noisy rolling KV cache kept per timestep, never refreshed with a clean
    forward (papernotes note, 关键设计 2 "History Corrupt"; gitcode blog,
    question 4);
  * timestep forcing: the cache read at step t_i holds K/V computed at t_i
    (papernotes note, 关键设计 4; gitcode blog, question 6);
  * Rolling RoPE: the sink frame's temporal position is re-offset each block so
    its distance to the active block is constant (papernotes note, 关键设计 3;
    admirer.cn article, "滾動位置編碼");
  * Adaptive Attention Sink: the first generated latent replaces the reference
    sink once (papernotes note, 关键设计 3; gitcode blog, question 5);
  * per-token RMS pre-norm of every sublayer input and of the head input
    (a reading: the pages give no layer internals; see oracle/norm.py);
  * flow-matching velocity v ~ x1 - x0 and an Euler step between the 4
    distilled timesteps (papernotes note, 损失函数 / L_FM);
  * the timestep-pipelined order of the 4 in-flight blocks (10100.com article,
    TPP figure caption; gitcode blog, question 6);
  * the clean-cache refresh ablation (oracle/schedule.py, oracle/stream.py),
    and per-row e4m3 quantization with the FP8 GEMM plus FP8 attention
    (oracle/fp8.py) for the operator-optimisation row (papernotes note, the
    paper's Table 3);
  * the full synthetic DiT block (oracle/dit.py): AdaLN-modulated attention
    and tanh-GELU FFN sub-blocks with gated residuals (a reading after the
    Wan-style block the model is built on; the pages give no internals).

Everything is fp64 numpy with a dict-indexed cache, an explicit mask matrix and
a naive softmax.  Where the pages are silent, each module states the reading it
takes in its own docstring (flow direction and timesteps in flow.py, the RoPE
pair layout and the sink offset in rope.py, the ring layout and eviction in
schedule.py, the FP8 scales in fp8.py, the block internals in dit.py).

Pins (tests/test_oracle_*.py): brute force on tiny inputs, SDPA on the visible
segments, softmax rows summing to 1, single-key passthrough, RoPE norm and
relative-position identities against a complex-number formulation, the Rolling
RoPE offset up to 10,000 blocks, (block, step) cache tags, the flow-matching
straight-line closed form, pipelined == sequential order with the sink fixed,
and closed forms of the layer with special weights.  Agreement with the real
14B Live Avatar model is parity unpinned: the pages give no weights, code or
worked example.
"""
from .rope import axis_frequencies, rope_rotate, block_positions, sink_positions
from .attention import block_causal_attention
from .flow import euler_step
from .norm import RMS_EPS, rms_norm
from .schedule import TickScheduler, index_state_layout
from .stream import OracleStream

__all__ = [
    "axis_frequencies", "rope_rotate", "block_positions", "sink_positions",
    "block_causal_attention", "euler_step", "rms_norm", "RMS_EPS", "TickScheduler", "index_state_layout",
    "OracleStream",
]
