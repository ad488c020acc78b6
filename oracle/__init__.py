"""CPU oracle (test infrastructure only): see oracle.py and oracle.c."""
