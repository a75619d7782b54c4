"""Write the expected velocity of the 30-block Wan 1.3B stack at 480P (32760 tokens) on
the sampled tokens, for the full-size stack parity test.

Calls only the oracle and the seeded input generator. The workload is the 1.3B stack of
"Wan: Open and Advanced Large-Scale Video Generative Models (Wan 2.1)" (section
"Diffusion Transformer", config table: dim 1536, 12 heads, FFN 8960, 30 layers) with one
rectified-flow velocity evaluation (section "训练方法": x_t = t x1 + (1 - t) x0, model
timestep 1000 t), seed 0. The oracle's float32-product / float64-reduction stack
(``dit_stack_f32``) evaluates every block on all tokens and the last block and the head
on the 256 sampled tokens of ``sample_rows`` (rows 0 and L-1 and the ragged last tile
included). Output: ``wan13b_480p_stack30_seed0_velocity_rows.npz`` beside this script,
with ``rows``, ``values`` ([256, 64]: each token's 16 channels x 2 x 2 outputs in
(c, ph, pw) order), the inputs' digest, and the run's time and thread count.

Usage: ``python tests/golden/make_stack30_velocity.py`` (about 20-40 minutes on 8 host
cores, ~8 GB of host memory).
"""
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from oracle import wan_oracle as O  # noqa: E402
from wan_inputs import WORKLOADS, input_digest, make_inputs, sample_rows  # noqa: E402

NAME = "wan13b_480p_stack30"
SEED = 0
OUT = os.path.join(HERE, f"{NAME}_seed{SEED}_velocity_rows.npz")


def main() -> None:
    import torch
    w = WORKLOADS[NAME]
    t0 = time.time()
    inp = make_inputs(w, seed=SEED, block_input=False)
    digest = input_digest(inp)
    rows = sample_rows(w.tokens)
    u = float(inp["u"][0])
    xt = O.flow_matching_input(inp["x1"][0], inp["noise"][0], u)
    print(f"inputs ready in {time.time() - t0:.0f} s; digest {digest[:16]}; u = {u:.6f}", flush=True)
    t1 = time.time()

    def progress(i):
        print(f"block {i + 1}/{w.n_blocks} done at {time.time() - t1:.0f} s", flush=True)

    values = O.dit_stack_f32(xt, 1000.0 * u, inp, inp["blocks"], inp["ctx"][0], w.heads, eps=w.eps,
                             freq_dim=w.freq_dim, rows=rows, progress=progress)
    seconds = time.time() - t1
    np.savez(OUT, rows=rows, values=np.asarray(values, dtype=np.float64), digest=np.array(digest),
             seconds=np.array(seconds), threads=np.array(torch.get_num_threads()), u=np.array(u))
    print(f"wrote {OUT}: {values.shape} values, {seconds:.0f} s on {torch.get_num_threads()} threads", flush=True)


if __name__ == "__main__":
    main()
