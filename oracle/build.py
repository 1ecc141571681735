"""Compile the C oracle (gcc + OpenMP) into oracle/_zq_oracle.so."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

if __name__ == "__main__":
    import oracle

    print(oracle.build(force=True))
