"""Run every oracle pin against the library given on the command line.

Prints a JSON list of failing pins. Used by test_oracle_mutants.py in a child
process, so that a mutant that crashes cannot take the test run down.
"""

import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import oracle as O  # noqa: E402
import oracle_pins as P  # noqa: E402

if __name__ == "__main__":
    lib = O.load(sys.argv[1])
    print(json.dumps(P.run_all(lib)))
