"""Write oracle_snapshot_small.json: the fp64 oracle (expanded definition) on the small
MLRA-4 workload (B=1, h=16, T=2048), heads 0..3.  Calls only oracle/ and synth/.

Run from the repository root:  python tests/golden/make_oracle_snapshot.py
"""
import json
import pathlib
import sys

ROOT = pathlib.Path(__file__).resolve().parents[2]
sys.path.insert(0, str(ROOT))

import oracle  # noqa: E402
import synth   # noqa: E402

wl = synth.WORKLOADS["small_mlra4_h16_t2k"]
inp = synth.make_inputs(wl)
heads = [0, 1, 2, 3]
out = oracle.decode_batch(inp, wl, heads=heads, seqs=[0], form="expanded")[0]
path = pathlib.Path(__file__).parent / "oracle_snapshot_small.json"
path.write_text(json.dumps({"workload": wl.name, "heads": heads, "out": out.tolist(),
                            "written_by": "tests/golden/make_oracle_snapshot.py"}, indent=0))
print("wrote", path)
