"""The ncu summaries under profiles/ name the commands that produced them; every
script those commands run must be a file of this repository, so that a capture
can be repeated from the committed tree."""
import glob
import json
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _commands(md: str):
    blocks = re.findall(r"```\n(.*?)```", md, flags=re.S)
    return [line for b in blocks for line in b.replace("\\\n", " ").splitlines() if "python" in line]


def test_profile_commands_run_committed_scripts():
    files = sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md")))
    assert files
    for f in files:
        cmds = _commands(open(f).read())
        assert cmds, f"{os.path.basename(f)} gives no command"
        for c in cmds:
            for script in re.findall(r"python\S*\s+(\S+\.py)", c):
                assert os.path.isfile(os.path.join(ROOT, script)), f"{os.path.basename(f)}: {script} is not in the tree"


def test_traffic_record_names_its_profile_and_sources():
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for kernel, r in rec.items():
        assert os.path.isfile(os.path.join(ROOT, r["profile"])), kernel
        for s in r["sources"]:
            assert os.path.isfile(os.path.join(ROOT, "sparse_attention_hyb_b200", "csrc", s)), (kernel, s)
        assert r["dram_bytes_per_launch"] > 0 and len(r["source_hash"]) == 16
