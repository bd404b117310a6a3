"""CPU oracle of the ISD step -- test infrastructure only (see isd_oracle.py)."""
