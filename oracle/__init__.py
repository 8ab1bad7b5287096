"""TEST INFRASTRUCTURE ONLY: the fp64 CPU oracle (see oracle.py and gdn_oracle.cpp)."""
