"""The calibrated threshold table: the one persistent artefact of the method.

"TEAL: Training-Free Activation Sparsity in Large Language Models", slide 8:
a site's threshold t_p is chosen once on calibration data for a target
sparsity and reused at inference. The table keeps the thresholds keyed by
(config, site, p, seed) in a small JSON file; values are stored as exact
hexadecimal floats (they are values of the calibration dtype, and -inf for
p = 0), so a reload gives the same bits. A missing entry is calibrated on the
GPU with sfx_calibrate_thresholds and added.
"""
from __future__ import annotations

import json
import os


def _key(config: str, site: str, p: float, seed) -> str:
    return json.dumps([str(config), str(site), float(p).hex(), str(seed)])


class ThresholdTable:
    """Thresholds keyed by (config, site, p, seed), saved as JSON."""

    VERSION = 1

    def __init__(self, path: str | None = None):
        self.path = path
        self.entries: dict[str, float] = {}
        if path and os.path.exists(path):
            self.load(path)

    def get(self, config, site, p, seed):
        return self.entries.get(_key(config, site, p, seed))

    def put(self, config, site, p, seed, t: float):
        self.entries[_key(config, site, p, seed)] = float(t)

    def calibrate(self, config, site, calib, ps, seed, ws=None):
        """Thresholds of `site` for each p in ps: from the table, else calibrated
        on `calib` (a [S x K] GPU tensor of the site's calibration draws)."""
        missing = [p for p in ps if self.get(config, site, p, seed) is None]
        if missing:
            from . import binding as sb
            for p, t in zip(missing, sb.sfx_calibrate_thresholds(calib, missing, ws=ws)):
                self.put(config, site, p, seed, t)
        return [self.get(config, site, p, seed) for p in ps]

    def save(self, path: str | None = None):
        path = path or self.path
        rows = [json.loads(k) + [v.hex()] for k, v in sorted(self.entries.items())]
        with open(path, "w") as f:
            json.dump({"version": self.VERSION, "key": ["config", "site", "p", "seed", "t"],
                       "entries": rows}, f, indent=1)

    def load(self, path: str):
        with open(path) as f:
            doc = json.load(f)
        if doc.get("version") != self.VERSION:
            raise ValueError(f"{path}: unknown threshold table version {doc.get('version')}")
        for config, site, p_hex, seed, t_hex in doc["entries"]:
            self.entries[_key(config, site, float.fromhex(p_hex), seed)] = float.fromhex(t_hex)
