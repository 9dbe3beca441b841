"""Child process of tests/test_gpu_timeout.py: runs decode calls through the library build
that PKV_LIB names (a test build whose first CTA withholds one stage, so one bounded wait
runs out), then one call that never reaches the withheld stage.  Writes the outputs and the
fault words it read to the directory given as argv[1]."""
import json
import os
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from paged_kv_cache_392_b200 import binding as B  # noqa: E402
from tests import timeout_cases as C  # noqa: E402


def main(out_dir):
    assert os.path.samefile(B.LIB_PATH, os.environ["PKV_LIB"])
    torch.cuda.set_device(0)
    B.device_faults(clear=True)
    res = {}
    for name in C.CASES:
        t0 = time.time()
        out = C.run(name, "cuda")
        torch.cuda.synchronize()
        res[name] = {"seconds": time.time() - t0, "faults": B.device_faults(clear=True)}
        np.save(os.path.join(out_dir, name + ".npy"), C.out_bits(out))
    with open(os.path.join(out_dir, "faults.json"), "w") as f:
        json.dump(res, f)


if __name__ == "__main__":
    main(sys.argv[1])
